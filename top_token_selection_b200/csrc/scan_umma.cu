// scan_umma.cu -- indexer scores on the 5th-generation tensor cores.
//
// Computes, for a block of P query rows (queries, proxy queries, or the
// members of one group) the indexer score against a stream of keys:
//     I(r, s) = sum_h w[r,h] * ReLU(q[r,h] . k[s])      (x q_scale * k_scale)
// (the dense indexer of "Sparse Attention의 Indexer", Fig. 1-2, in its
// multi-head form).  Two modes share one kernel:
//  * scan   -- keys 0..lim of the causal prefix, contiguous, loaded with tiled
//              TMA: the dense indexer, and the PIVOT proxy scan (abstract of
//              arXiv 2607.24593: one full-prefix scan per group, run with the
//              proxy as the query);
//  * gather -- the C candidate keys of the group, gathered row by row with
//              16-byte cp.async into the swizzled tile: PIVOT-Refine (same
//              abstract: every member re-scores the candidate set with its
//              own query).
//
// Mapping: keys on the MMA M axis (128 TMEM lanes), the P*H query heads on
// N (<= 256 columns).  Each epilogue thread owns one key and reduces its
// lane's columns over heads in registers -- no shuffles.  The query block is
// loaded once per work item and stays in shared memory; key tiles stream
// through a TMA ring.  Accumulators are double-buffered in TMEM (2 x 256
// columns) so the epilogue of tile i overlaps the MMAs of tile i+1.
//
// Warp roles.  Warp 0 loads (one lane issuing TMA in scan mode; all 32 lanes
// copying in gather mode, with warp 18 as a second copier), warp 1 allocates
// TMEM and issues tcgen05.mma, and warps 2-17 reduce, four per TMEM lane
// quarter: a block of 256 / H rows (N = 256), so at H = 64 each epilogue
// warp owns one row.  The block's halved head weights sit in shared memory
// (read as float4 broadcasts): four warps per quarter with 64 weights each in
// registers do not fit the 96 registers five warps a sub-partition leave.
#include "common.cuh"
#include "kernels.h"

namespace pivot {

// Warp layout: warp 0 loads, warp 1 issues the MMAs, warps 2-17 run the
// epilogue -- four per TMEM lane quarter, blocks of 256 / H rows (one row a
// warp at H = 64), the rows' halved head weights in shared memory -- and in
// gather mode warp 18 copies candidates beside warp 0.  Registers are per SM
// sub-partition (16K each; warp w runs on sub-partition w % 4): 18 or 19
// warps put five on one, so 96 registers a thread.
template <bool GATHER> struct EpiShape {
    static constexpr int GROUPS = 4;
    static constexpr int WARPS = 4 * GROUPS;                  // 16
    static constexpr int WARP2 = GATHER ? 2 + WARPS : -1;     // second copying warp
    static constexpr int THREADS = (2 + WARPS + (GATHER ? 1 : 0)) * 32;   // 576 / 608
    static constexpr int MAXREG = 96;
};
static_assert(5 * 32 * EpiShape<false>::MAXREG <= 16384 && 5 * 32 * EpiShape<true>::MAXREG <= 16384,
              "register file of a sub-partition");

__device__ __forceinline__ int scan_row_lim(const ScanParams& p, int r, bool& ok) {
    ok = true;
    switch (p.kind) {
        case SCAN_PREFILL_DENSE:
            return r;
        case SCAN_PREFILL_PROXY: {
            int e = (r + 1) * p.g;
            return (e < p.L ? e : p.L) - 1;
        }
        case SCAN_DECODE_DENSE: {
            int b = r / p.Gm, m = r % p.Gm;
            int n = p.cache_len[b];
            if (n < p.Gm || n > p.maxlen) { ok = false; return -1; }
            return n - p.Gm + m;
        }
        case SCAN_VARLEN_DENSE:
            return seg_dense_lim(p.seg, r);
        case SCAN_VARLEN_PROXY:
            return seg_proxy_lim(p.seg, p.g, r);
        default: {  // SCAN_DECODE_PROXY
            int n = p.cache_len[r];
            if (n < 1 || n > p.maxlen) { ok = false; return -1; }
            return n - 1;
        }
    }
}

__device__ __forceinline__ int scan_key_base(const ScanParams& p, int r) {
    if (p.kind == SCAN_DECODE_DENSE) return (r / p.Gm) * p.maxlen;
    if (p.kind == SCAN_DECODE_PROXY) return r * p.maxlen;
    return 0;
}

struct ItemInfo {
    int rows, row_first, t0, t1, keybase, maxlim;
    int chunk;             // scan mode: the item's chunk of key tiles
    int ncand;             // gather mode: candidates scored (C, or the group's adaptive count)
    int nkeys;             // gather mode: key rows of the item's sequence
    const int32_t* cand;   // gather mode: this group's candidate row
    bool valid;
};

// Scan mode: item i = (row block, chunk of key tiles); items whose chunk
// starts beyond the block's causal extent are empty.  Prefill launches number
// their items chunk by chunk (every row block's first chunk, then every
// block's second, ...): item i runs on CTA i mod grid, so numbering block by
// block gave CTA c only the chunks congruent to c modulo gcd(grid, chunks a
// block): with four chunks a block and 148 CTAs, a quarter of the CTAs got
// every block's first chunk while another quarter only got the fourth
// chunks of the longest rows.  Decode launches (few row blocks of
// ragged lengths) keep the block-by-block numbering.
// Gather mode: item i = (group, block of that group's member rows); the
// tiles cover the C candidates.  Every role walks the same item sequence.
template <bool GATHER>
__device__ __forceinline__ ItemInfo scan_item(const ScanParams& p, int item) {
    ItemInfo it;
    if constexpr (!GATHER) {
        int chunk;
        if (p.row_list) {
            // one listed row per block; slots past the device count are empty
            const int slot = item / p.items_per_block;
            chunk = item % p.items_per_block;
            if ((uint32_t)slot >= *p.row_count) {
                it.valid = false;
                it.rows = 0;
                it.row_first = p.row0;
                it.t0 = it.t1 = 0;
                it.maxlim = -1;
                it.nkeys = 0;
                it.keybase = 0;
                it.chunk = chunk;
                it.cand = nullptr;
                return it;
            }
            it.row_first = p.row_list[slot];
            it.rows = 1;
            it.keybase = scan_key_base(p, it.row_first);
        } else if (p.kind == SCAN_VARLEN_DENSE || p.kind == SCAN_VARLEN_PROXY) {
            // blocks never straddle two sequences: each is one sequence's;
            // rows outside the launch's [row0, row0 + nrows) are dropped
            const SegItem si = seg_scan_item(
                p.seg, p.kind == SCAN_VARLEN_DENSE ? p.seg.tok : p.seg.grp, p.P, p.row0, p.nrows, item);
            chunk = si.chunk;
            it.row_first = si.first;
            it.rows = si.rows;
            it.keybase = p.seg.tok[si.b];
            if (it.rows <= 0) {
                it.valid = false;
                it.t0 = it.t1 = 0;
                it.maxlim = -1;
                it.nkeys = 0;
                it.chunk = chunk;
                it.cand = nullptr;
                return it;
            }
        } else {
            int blk;
            if (p.kind == SCAN_PREFILL_DENSE || p.kind == SCAN_PREFILL_PROXY) {
                const int nblocks = p.nitems / p.items_per_block;   // items_per_block >= 1
                chunk = item / nblocks;
                blk = item % nblocks;
            } else {
                blk = item / p.items_per_block;
                chunk = item % p.items_per_block;
            }
            it.row_first = p.row0 + blk * p.P;
            const int rows = p.row0 + p.nrows - it.row_first;
            it.rows = rows < p.P ? rows : p.P;
            it.keybase = scan_key_base(p, it.row_first);
        }
        bool ok;
        const int maxlim = scan_row_lim(p, it.row_first + it.rows - 1, ok);
        it.maxlim = ok ? maxlim : -1;
        it.nkeys = 0;
        it.chunk = chunk;
        // key tiles of the block's longest prefix (sample scan: every
        // key_tile_stride-th of them)
        const int kts = p.key_tile_stride > 1 ? p.key_tile_stride : 1;
        const int nt = ok ? ((maxlim + 1 + 127) / 128 + kts - 1) / kts : 0;
        it.t0 = chunk * p.tiles_per_item;
        it.t1 = it.t0 + p.tiles_per_item < nt ? it.t0 + p.tiles_per_item : nt;
        it.valid = it.t0 < nt;
        it.cand = nullptr;
    } else {
        const int grp = p.cand_base + item / p.items_per_block;
        const int mb = item % p.items_per_block;
        if (p.kind == SCAN_VARLEN_DENSE) {   // packed group of a ragged batch
            const SegItem si = seg_refine_item(p.seg, p.gsize, p.P, grp, mb, p.row0, p.nrows);
            it.row_first = si.first;
            it.rows = si.rows;
            it.keybase = p.seg.tok[si.b];
            it.nkeys = p.seg.tok[si.b + 1] - p.seg.tok[si.b];
        } else {
            const int gstart = grp * p.gsize;
            int first = gstart + mb * p.P;
            int end = first + p.P;
            if (end > gstart + p.gsize) end = gstart + p.gsize;
            if (first < p.row0) first = p.row0;
            if (end > p.row0 + p.nrows) end = p.row0 + p.nrows;
            it.row_first = first;
            it.rows = end - first;
            it.keybase = p.kind == SCAN_DECODE_DENSE ? grp * p.maxlen : 0;
            it.nkeys = p.nkeys;
        }
        it.maxlim = it.nkeys - 1;
        it.chunk = 0;
        it.t0 = 0;
        // adaptive C: only the group's first ncand candidates are scored
        it.ncand = p.C;
        if (p.cand_count) {
            const int c = p.cand_count[grp - p.cand_base];
            it.ncand = c < 0 ? 0 : (c < p.C ? c : p.C);
        }
        it.t1 = (it.ncand + 127) / 128;
        it.valid = it.rows > 0 && it.t1 > 0;
        it.cand = p.cand + (size_t)(grp - p.cand_base) * p.C;
    }
    return it;
}

template <int KIND, int HEADS, int ROWB, bool GATHER, bool FILTER>
__global__ void __maxnreg__(EpiShape<GATHER>::MAXREG)
    index_umma_kernel(const __grid_constant__ CUtensorMap tmap_k,
                      const __grid_constant__ CUtensorMap tmap_q, const ScanParams p) {
    constexpr int KBLK = ROWB / 128;           // 128-byte K blocks per row
    constexpr int KSTEPS = ROWB / 32;          // one MMA consumes 32 bytes of K
    constexpr int A_BYTES = 128 * ROWB;        // one key tile
    constexpr int B_SLOT = 256 * ROWB;         // query block, N <= 256 rows
    constexpr int STAGES = ROWB == 128 ? 6 : 3;
    constexpr int PMAX = 256 / HEADS;
    constexpr int EPI_GROUPS = EpiShape<GATHER>::GROUPS;
    constexpr int EPI_WARPS = EpiShape<GATHER>::WARPS;
    constexpr int GATHER_WARP2 = EpiShape<GATHER>::WARP2;
    constexpr int FIRST_EPI = 2;
    constexpr int TCOLS = 32;                   // TMEM columns a load at H >= 32
    constexpr uint32_t FMT = KIND == KIND_F8 ? 0u : (KIND == KIND_F16 ? 1u : 2u);

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sB = smem;                                   // 2 slots
    uint8_t* sA = smem + 2 * B_SLOT;                      // STAGES tiles
    uint64_t* bars = reinterpret_cast<uint64_t*>(sA + STAGES * A_BYTES);
    uint64_t* full = bars;                                // [STAGES]
    uint64_t* empty = bars + STAGES;                      // [STAGES]
    uint64_t* bfull = bars + 2 * STAGES;                  // [2]
    uint64_t* bempty = bfull + 2;                         // [2]
    uint64_t* accfull = bempty + 2;                       // [2]
    uint64_t* accempty = accfull + 2;                     // [2]
    uint64_t* drain = accempty + 2;                       // [1]
    // barriers take at most 2*6+9 = 21 words of the 256 bytes reserved
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(bars) + 256);
    float* w_s = reinterpret_cast<float*>(tmem_holder + 4);   // [256], 16-byte aligned
    float* sq_s = w_s + 256;                                   // [PMAX]
    int* lim_s = reinterpret_cast<int*>(sq_s + PMAX);          // [PMAX]

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int N = p.P * HEADS;
    // row-list mode: only the listed rows' items (the count is read once)
    int nitems = p.nitems;
    if (p.row_list) {
        const long long lim = (long long)(*p.row_count) * p.items_per_block;
        if (lim < nitems) nitems = (int)lim;
    }

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            // gather mode: both gathering warps publish each tile
            mbar_init(&full[i], GATHER ? 2 : 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bfull[i], 1);
            mbar_init(&bempty[i], 1);
            mbar_init(&accfull[i], 1);
            mbar_init(&accempty[i], EPI_WARPS);   // one arrive per epilogue warp
        }
        mbar_init(drain, 1);
        fence_barrier_init();
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_q);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    if (warp < FIRST_EPI || (GATHER && warp == GATHER_WARP2)) {
        if (warp == 0 || (GATHER && warp == GATHER_WARP2)) {
            // ------------------------------------------------------- producer
            if constexpr (!GATHER) {
                if (warp == 0) {
                // Scan mode: lane 0 streams contiguous key tiles with tiled TMA.
                if (lane == 0) {
                    int stage = 0;
                    uint32_t phase = 0;
                    int nit = 0;
                    // parity of the last load issued per stage / query slot (-1:
                    // none), so every load can be waited for before the CTA exits
                    int last_a[STAGES], last_b[2] = {-1, -1};
                    for (int i = 0; i < STAGES; ++i) last_a[i] = -1;
                    bool aborted = false;
                    for (int item = blockIdx.x; item < nitems && !aborted; item += gridDim.x) {
                        ItemInfo it = scan_item<GATHER>(p, item);
                        if (!it.valid) continue;
                        const int slot = nit & 1;
                        const uint32_t bph = (nit >> 1) & 1;
                        if (!mbar_wait(&bempty[slot], bph ^ 1)) { aborted = true; break; }
                        mbar_arrive_expect_tx(&bfull[slot], (uint32_t)(N * ROWB));
                        last_b[slot] = (int)bph;
                        const int qrow = (it.row_first - p.qrow_base) * HEADS;
                        for (int kb = 0; kb < KBLK; ++kb)
                            tma_load_2d(sB + slot * B_SLOT + kb * (N * 128), &tmap_q, &bfull[slot],
                                        kb * (128 / p.esize), qrow);
                        for (int t = it.t0; t < it.t1; ++t) {
                            if (!mbar_wait(&empty[stage], phase ^ 1)) { aborted = true; break; }
                            mbar_arrive_expect_tx(&full[stage], (uint32_t)A_BYTES);
                            last_a[stage] = (int)phase;
                            const int kt = p.key_tile_stride > 1 ? t * p.key_tile_stride : t;
                            for (int kb = 0; kb < KBLK; ++kb)
                                tma_load_2d(sA + stage * A_BYTES + kb * (128 * 128), &tmap_k,
                                            &full[stage], kb * (128 / p.esize), it.keybase + kt * 128);
                            if (++stage == STAGES) { stage = 0; phase ^= 1; }
                        }
                        ++nit;
                    }
                    // Every load issued lands before the CTA may exit (only the
                    // producer arrives on these barriers, so the last phase stays).
                    for (int i = 0; i < STAGES; ++i)
                        if (last_a[i] >= 0) mbar_wait(&full[i], (uint32_t)last_a[i]);
                    for (int i = 0; i < 2; ++i)
                        if (last_b[i] >= 0) mbar_wait(&bfull[i], (uint32_t)last_b[i]);
                }
                }
            } else {
                // Gather mode: two warps copy each tile's 128 candidate key rows
                // (warp 0 rows 0-63, warp 18 rows 64-127) with 16-byte cp.async
                // straight into the swizzled tile layout.  Each publishes its half
                // of a tile (an arrive on full[stage], which expects both) once
                // its copies have landed and been fenced for the tensor cores; up
                // to GDEPTH tiles are in flight per warp.  Warp 0 alone loads the
                // query blocks.  Neither warp blocks while holding an unpublished
                // tile older than the one it waits for: warp 0 publishes the
                // tiles of item nit - 2 before waiting for its query slot, and a
                // ring stage a warp waits on was last used by a tile older than
                // all of that warp's pending ones (STAGES > GDEPTH).
                const bool lead = warp == 0;
                const int jb = lead ? 0 : 2;   // row groups j of this warp (rows j * 32 + lane)
                constexpr int GDEPTH = STAGES > 3 ? 3 : STAGES - 1;   // deeper was slower
                static_assert(STAGES > GDEPTH && GDEPTH >= 1, "the ring must outrun the copies");
                const uint8_t* kbytes = static_cast<const uint8_t*>(p.kbase);
                int stage = 0;
                uint32_t phase = 0;
                int nit = 0;
                int pend[GDEPTH] = {0};       // stages of the tiles in flight, oldest first
                int pend_it[GDEPTH] = {0};    // and the item (in this CTA's order) of each
                int npend = 0;
                int last_b[2] = {-1, -1};
                bool aborted = false;
                auto publish_oldest = [&]() {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full[pend[0]]);
                    for (int i = 1; i < npend; ++i) {
                        pend[i - 1] = pend[i];
                        pend_it[i - 1] = pend_it[i];
                    }
                    --npend;
                };
                for (int item = blockIdx.x; item < nitems && !aborted; item += gridDim.x) {
                    ItemInfo it = scan_item<GATHER>(p, item);
                    if (!it.valid) continue;
                    const int slot = nit & 1;
                    const uint32_t bph = (nit >> 1) & 1;
                    // The query slot frees once the MMAs of item nit - 2 are done,
                    // which needs every tile of that item published: land and
                    // publish what is in flight if any of it is that old (items
                    // shorter than the copy depth).
                    if (lead) {
                        if (npend > 0 && pend_it[0] <= nit - 2) {
                            cp_async_wait<0>();
                            while (npend > 0) publish_oldest();
                        }
                        if (!__all_sync(0xffffffffu, mbar_wait(&bempty[slot], bph ^ 1))) {
                            aborted = true;
                            break;
                        }
                        if (lane == 0) {
                            mbar_arrive_expect_tx(&bfull[slot], (uint32_t)(N * ROWB));
                            const int qrow = (it.row_first - p.qrow_base) * HEADS;
                            for (int kb = 0; kb < KBLK; ++kb)
                                tma_load_2d(sB + slot * B_SLOT + kb * (N * 128), &tmap_q, &bfull[slot],
                                            kb * (128 / p.esize), qrow);
                        }
                        last_b[slot] = (int)bph;
                    }
                    // candidate positions of this warp's rows of a tile: lane l
                    // holds slots l + 32 (jb + j), read one tile ahead so no copy
                    // waits on them
                    auto tile_pos = [&](int t, int (&pp)[2]) {
    #pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const int slot_r = t * 128 + (jb + j) * 32 + lane;
                            pp[j] = slot_r < it.ncand ? ld_nc_early(it.cand + slot_r) : -1;
                        }
                    };
                    int cur[2], nxt[2];
                    tile_pos(it.t0, nxt);
                    for (int t = it.t0; t < it.t1; ++t) {
    #pragma unroll
                        for (int j = 0; j < 2; ++j) cur[j] = nxt[j];
                        if (t + 1 < it.t1) tile_pos(t + 1, nxt);
                        if (!__all_sync(0xffffffffu, mbar_wait(&empty[stage], phase ^ 1))) {
                            aborted = true;
                            break;
                        }
                        const uint32_t dst = smem_u32(sA + stage * A_BYTES);
                        // Eight lanes copy one row together: in instruction i
                        // lanes 8q .. 8q + 7 take the 16-byte chunks c = lane % 8
                        // of this warp's row 4i + q, whose position the lane that
                        // read it passes by a shuffle, so each instruction reads
                        // four whole 128-byte lines (one line a chunk per lane had
                        // each instruction touch 32 lines: 256-byte bf16 rows took
                        // 18.1 ms of Refine scan at L = 64K, C = 8192, now 11.4).
                        // Chunk c of row r sits at (r / 8) 1024 + (r % 8) 128 +
                        // ((c ^ r % 8) 16), the 128-byte swizzle of a 1024-byte
                        // aligned tile.
                        {
                            const uint32_t c = (uint32_t)(lane & 7);
    #pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const int rl = 4 * i + (lane >> 3);
                                const int pos = __shfl_sync(0xffffffffu, cur[i >> 3], rl & 31);
                                const int r = jb * 32 + rl;
                                const size_t row = (size_t)(it.keybase + ((pos >= 0 && pos < it.nkeys) ? pos : 0));
                                const uint8_t* src = kbytes + row * ROWB + c * 16;
                                const uint32_t x = (uint32_t)(r & 7);
                                const uint32_t d = dst + (uint32_t)(r >> 3) * 1024u + x * 128u + ((c ^ x) << 4);
    #pragma unroll
                                for (int kb = 0; kb < KBLK; ++kb)
                                    cp_async16_ca(d + kb * (128 * 128), src + kb * 128);
                            }
                        }
                        cp_async_commit();
                        pend_it[npend] = nit;
                        pend[npend++] = stage;
                        if (npend == GDEPTH) {
                            cp_async_wait<GDEPTH - 1>();
                            publish_oldest();
                        }
                        if (++stage == STAGES) { stage = 0; phase ^= 1; }
                    }
                    ++nit;
                }
                // publish (or, after an abort, just land) every tile still in flight
                cp_async_wait<0>();
                while (npend > 0) publish_oldest();
                if (lead && lane == 0)
                    for (int i = 0; i < 2; ++i)
                        if (last_b[i] >= 0) mbar_wait(&bfull[i], (uint32_t)last_b[i]);
            }
        } else if (warp == 1) {
            // ------------------------------------------------------------ MMA
            if (lane == 0) {
                const uint32_t idesc = make_idesc(FMT, 128, (uint32_t)N);
                int stage = 0;
                uint32_t phase = 0;
                int nit = 0, ntile = 0;
                bool aborted = false;
                for (int item = blockIdx.x; item < nitems && !aborted; item += gridDim.x) {
                    ItemInfo it = scan_item<GATHER>(p, item);
                    if (!it.valid) continue;
                    const int slot = nit & 1;
                    const uint32_t bph = (nit >> 1) & 1;
                    if (!mbar_wait(&bfull[slot], bph)) { aborted = true; break; }
                    const uint32_t bbase = smem_u32(sB + slot * B_SLOT);
                    for (int t = it.t0; t < it.t1; ++t) {
                        const int acc = ntile & 1;
                        const uint32_t aph = (ntile >> 1) & 1;
                        if (!mbar_wait(&accempty[acc], aph ^ 1)) { aborted = true; break; }
                        if (!mbar_wait(&full[stage], phase)) { aborted = true; break; }
                        tc_fence_after();
                        const uint32_t abase = smem_u32(sA + stage * A_BYTES);
                        const uint32_t dcol = tmem_base + (uint32_t)(acc * 256);
    #pragma unroll
                        for (int ks = 0; ks < KSTEPS; ++ks) {
                            const int kb = ks / 4, kin = ks % 4;
                            const uint64_t ad = smem_desc_k_sw128(abase + kb * (128 * 128) + kin * 32);
                            const uint64_t bd = smem_desc_k_sw128(bbase + kb * (N * 128) + kin * 32);
                            umma_ss<KIND>(dcol, ad, bd, idesc, ks > 0 ? 1u : 0u);
                        }
                        umma_commit(&empty[stage]);
                        umma_commit(&accfull[acc]);
                        if (++stage == STAGES) { stage = 0; phase ^= 1; }
                        ++ntile;
                    }
                    umma_commit(&bempty[slot]);
                    ++nit;
                }
                // Drain: wait until every MMA issued has completed.
                umma_commit(drain);
                mbar_wait(drain, 0);
            }
        }
    } else {
        // ------------------------------------------------------- epilogue
        // EPI_GROUPS warps per TMEM lane quarter.  With H >= 32 the rows of
        // the block are split between the groups (each row's H columns are
        // reduced by one thread; the halved head weights in registers in
        // gather mode, in shared memory in scan mode); with H < 32 the first
        // group does all rows in 32-column chunks (weights from shared
        // memory) and the others only keep step.
        const int e = warp - FIRST_EPI;           // 0..EPI_WARPS-1
        const int quarter = warp & 3;             // TMEM lane quarter of this warp
        const int grp = e >> 2;                   // 0..EPI_GROUPS-1
        const int key_in_tile = quarter * 32 + lane;
        const int et = e * 32 + lane;
        int r_lo = 0, r_hi = 0;
        if constexpr (HEADS >= 32) {
            const int Pg = (p.P + EPI_GROUPS - 1) / EPI_GROUPS;   // <= 64 / HEADS
            r_lo = grp * Pg < p.P ? grp * Pg : p.P;
            r_hi = r_lo + Pg < p.P ? r_lo + Pg : p.P;
        } else {
            r_hi = grp == 0 ? p.P : 0;
        }
        constexpr int RROWS = HEADS >= 32 ? 64 / HEADS : 1;      // rows per warp at most
        int lim_r[RROWS];
        float sq_r[RROWS];
        float tf_r[RROWS];    // filter mode: scores >= tf_r are kept
        uint32_t nkept[RROWS];  // filter mode: this warp's survivors of the item, per row
        int ntile = 0;
        const int kts = p.key_tile_stride > 1 ? p.key_tile_stride : 1;
        constexpr bool filter = FILTER && !GATHER && HEADS >= 32;
        // Once a wait runs out the warp stops touching TMEM and memory but
        // keeps walking the items, so the named barriers shared by the
        // epilogue warps are always reached.
        bool aborted = false;
        for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
            ItemInfo it = scan_item<GATHER>(p, item);
            if (!it.valid) continue;
            // gather mode: every candidate slot is written (the selection
            // drops empty slots and positions after the member)
            auto row_lim = [&](int pr) -> int {
                if (pr >= it.rows) return -1;
                if (GATHER) return 0x7fffffff;
                bool ok = true;
                const int lim = scan_row_lim(p, it.row_first + pr, ok);
                return ok ? lim : -1;
            };
            auto row_sq = [&](int pr) -> float {
                return (p.q_scale && pr < it.rows) ? p.q_scale[it.row_first + pr - p.qrow_base]
                                                   : 1.0f;
            };
            if constexpr (HEADS >= 32) {
                // the block's halved head weights, P x H <= 256 floats
                // (w * max(0, x) == (w / 2) * (x + |x|) exactly)
                named_bar_sync(1, EPI_WARPS * 32);
                for (int i = et; i < p.P * HEADS; i += EPI_WARPS * 32) {
                    const int pr = i / HEADS;
                    w_s[i] = pr < it.rows
                                 ? 0.5f * p.w[(size_t)(it.row_first + pr - p.qrow_base) * HEADS +
                                              i % HEADS]
                                 : 0.0f;
                }
                named_bar_sync(1, EPI_WARPS * 32);
                // this warp's rows: limits and query scales in registers
#pragma unroll
                for (int lr = 0; lr < RROWS; ++lr) {
                    const int pr = r_lo + lr;
                    const bool live = pr < r_hi && pr < it.rows;
                    lim_r[lr] = pr < r_hi ? row_lim(pr) : -1;
                    sq_r[lr] = row_sq(pr);
                    tf_r[lr] = -INFINITY;
                    nkept[lr] = 0;
                    if (filter && live && p.bound) {
                        const uint32_t T = p.bound[it.row_first + pr - p.row0];
                        if (T > 0x00800000u) tf_r[lr] = key_to_float(T);
                    }
                }
            } else {
                named_bar_sync(1, EPI_WARPS * 32);
                // The tables span all 256 columns / PMAX rows: a TMEM load
                // covers 32 columns even when N is 16, and the columns past N
                // must map to masked rows (lim -1) with zero weights.
                for (int i = et; i < 256; i += EPI_WARPS * 32) {
                    const int pr = i / HEADS;
                    w_s[i] = (i < N && pr < it.rows)
                                 ? p.w[(size_t)(it.row_first + pr - p.qrow_base) * HEADS + i % HEADS]
                                 : 0.0f;
                }
                for (int pr = et; pr < PMAX; pr += EPI_WARPS * 32) {
                    lim_s[pr] = row_lim(pr);
                    sq_s[pr] = row_sq(pr);
                }
                named_bar_sync(1, EPI_WARPS * 32);
            }
            // Key scale of this thread's key in tile t (1 where none), read a
            // tile ahead.  Gather mode stores its scores without the key
            // scale (the candidate selection multiplies it in): reading the
            // candidate's position and then its scale here put two dependent
            // loads on every tile and halved the rate.
            auto key_scale = [&](int t) -> float {
                if (GATHER || !p.k_scale) return 1.0f;
                const int s_t = t * kts * 128 + key_in_tile;
                return s_t <= it.maxlim ? ld_nc_early(p.k_scale + it.keybase + s_t) : 1.0f;
            };
            float sk_next = key_scale(it.t0);
            for (int t = it.t0; t < it.t1; ++t) {
                const int acc = ntile & 1;
                const uint32_t aph = (ntile >> 1) & 1;
                ++ntile;
                const float sk = sk_next;                  // prefetched a tile ahead
                if (t + 1 < it.t1) sk_next = key_scale(t + 1);
                if (aborted) continue;
                const bool got = mbar_wait(&accfull[acc], aph);
                if (!__all_sync(0xffffffffu, got)) { aborted = true; continue; }
                tc_fence_after();
                // s: the output column (key position in scan mode, sample
                // index in the sample scan, candidate slot in gather mode);
                // spos: the key position the causal limit applies to
                const int s = t * 128 + key_in_tile;
                const int spos = kts > 1 ? t * kts * 128 + key_in_tile : s;
                const bool col_ok = GATHER ? (s < it.ncand) : true;
                const uint32_t taddr =
                    tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * 256);
                if constexpr (HEADS >= 32) {
#pragma unroll
                    for (int lr = 0; lr < RROWS; ++lr) {
                        const int pr = r_lo + lr;
                        if (pr >= r_hi) break;
                        // four packed partial sums (two multiply-adds per instruction)
                        uint64_t a[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) a[j] = 0ull;
#pragma unroll
                        for (int c = 0; c < HEADS / TCOLS; ++c) {
                            float v[TCOLS];
                            tmem_ld32(taddr + (uint32_t)(pr * HEADS + c * TCOLS), v);
                            tmem_ld_wait();
                            // x + |x| = 2 max(0, x): one add on the FMA pipe
                            // instead of a half-rate max on the ALU pipe; four
                            // weights a broadcast load (every lane the same row)
                            const float4* w4 =
                                reinterpret_cast<const float4*>(w_s + pr * HEADS + c * TCOLS);
#pragma unroll
                            for (int i = 0; i < TCOLS / 4; ++i) {
                                const float4 wv = w4[i];
                                a[(2 * i) & 3] =
                                    ffma2(pack2(v[4 * i] + fabsf(v[4 * i]),
                                                v[4 * i + 1] + fabsf(v[4 * i + 1])),
                                          pack2(wv.x, wv.y), a[(2 * i) & 3]);
                                a[(2 * i + 1) & 3] =
                                    ffma2(pack2(v[4 * i + 2] + fabsf(v[4 * i + 2]),
                                                v[4 * i + 3] + fabsf(v[4 * i + 3])),
                                          pack2(wv.z, wv.w), a[(2 * i + 1) & 3]);
                            }
                        }
                        float lo[4], hi[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) unpack2(a[j], lo[j], hi[j]);
                        const float rowsum = ((lo[0] + hi[0]) + (lo[1] + hi[1])) +
                                             ((lo[2] + hi[2]) + (lo[3] + hi[3]));
                        const float score = rowsum * sq_r[lr] * sk;
                        if constexpr (filter) {
                            // survivors only, appended to this warp's own
                            // sub-region of the row's chunk (its TMEM lane
                            // quarter: 32 keys of every tile of the item),
                            // counted in a register; the keep-everything
                            // rescan of listed rows writes each key at its
                            // own position instead
                            const bool keep = spos <= lim_r[lr] - p.lim_shift &&
                                              score >= tf_r[lr];
                            const unsigned m = __ballot_sync(0xffffffffu, keep);
                            if (keep) {
                                const uint32_t at = nkept[lr] + __popc(m & ((1u << lane) - 1u));
                                const uint64_t key =
                                    ((uint64_t)ordered_key(score) << 32) |
                                    (uint64_t)(0xFFFFFFFFu - (uint32_t)spos);
                                uint64_t* row = p.surv + (size_t)(it.row_first + pr - p.row0) *
                                                             p.surv_stride;
                                if (p.row_list) {
                                    if (PIVOT_CHECK(spos < p.surv_stride)) row[spos] = key;
                                } else if (PIVOT_CHECK(at < (uint32_t)(p.tiles_per_item * 32))) {
                                    row[(size_t)it.chunk * (p.tiles_per_item * 128) +
                                        (size_t)quarter * (p.tiles_per_item * 32) + at] = key;
                                }
                            }
                            nkept[lr] += __popc(m);
                        } else if (col_ok && spos <= lim_r[lr] && PIVOT_CHECK(s < p.S_stride)) {
                            // streaming store: keep L2 for the keys
                            __stcs(p.S + (size_t)(it.row_first + pr - p.row0) * p.S_stride + s,
                                   score);
                        }
                    }
                } else {
                    if (r_hi > 0) {
                        float rowacc = 0.0f;
                        float v[32];
#pragma unroll 1
                        for (int c0 = 0; c0 < N; c0 += 32) {
                            tmem_ld32(taddr + c0, v);
                            tmem_ld_wait();
#pragma unroll
                            for (int i = 0; i < 32; ++i) {
                                rowacc = fmaf(w_s[c0 + i], fmaxf(v[i], 0.0f), rowacc);
                                if ((i + 1) % HEADS == 0) {
                                    const int pr = (c0 + i) / HEADS;
                                    if (col_ok && spos <= lim_s[pr])
                                        __stcs(p.S + (size_t)(it.row_first + pr - p.row0) *
                                                         p.S_stride + s,
                                               rowacc * sq_s[pr] * sk);
                                    rowacc = 0.0f;
                                }
                            }
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&accempty[acc]);
            }
            if constexpr (filter) {
                // this warp's survivor counts of the item, one per row it owns
                if (lane == 0 && !aborted && !p.row_list) {
#pragma unroll
                    for (int lr = 0; lr < RROWS; ++lr) {
                        const int pr = r_lo + lr;
                        if (pr < r_hi && pr < it.rows)
                            p.surv_count[((size_t)(it.row_first + pr - p.row0) * p.nchunks +
                                          it.chunk) * 4 + quarter] = nkept[lr];
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

int scan_smem_bytes(int row_bytes) {
    const int stages = row_bytes == 128 ? 6 : 3;
    const int pmax = 64;
    return 1024 /*align slack*/ + 2 * 256 * row_bytes + stages * 128 * row_bytes +
           256 /*barriers*/ + 16 /*TMEM address*/ + 256 * 4 + pmax * 8;
}

// The epilogue's warp groups (four in scan mode, three in gather mode) take
// ceil(P / groups) rows each, with room for 64 / HEADS rows' weights in
// registers at HEADS >= 32, and PMAX rows' tables in shared memory below:
// larger blocks are refused.
inline bool epilogue_fits(int P, int heads, int groups) {
    if (P < 1 || P * heads > 256) return false;
    return heads >= 32 ? (P + groups - 1) / groups <= 64 / heads : true;
}

template <int KIND, int HEADS, int ROWB, bool GATHER, bool FILTER>
static cudaError_t launch_one(const CUtensorMap& tk, const CUtensorMap& tq, const ScanParams& p,
                              int grid, cudaStream_t stream) {
    auto kfn = index_umma_kernel<KIND, HEADS, ROWB, GATHER, FILTER>;
    const int smem = scan_smem_bytes(ROWB);
    cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kfn<<<grid, EpiShape<GATHER>::THREADS, smem, stream>>>(tk, tq, p);
    return cudaGetLastError();
}

template <int KIND, int HEADS, bool GATHER>
static cudaError_t launch_heads(const CUtensorMap& tk, const CUtensorMap& tq, const ScanParams& p,
                                int row_bytes, int grid, cudaStream_t stream) {
    if (!epilogue_fits(p.P, HEADS, EpiShape<GATHER>::GROUPS)) return cudaErrorInvalidValue;
    // the fused selection runs in the register-resident epilogue (H >= 32)
    const bool filter = !GATHER && p.surv != nullptr;
    if (filter && HEADS < 32) return cudaErrorInvalidValue;
    if constexpr (!GATHER && HEADS >= 32) {
        if (filter)
            return row_bytes == 128 ? launch_one<KIND, HEADS, 128, false, true>(tk, tq, p, grid, stream)
                                    : launch_one<KIND, HEADS, 256, false, true>(tk, tq, p, grid, stream);
    }
    return row_bytes == 128 ? launch_one<KIND, HEADS, 128, GATHER, false>(tk, tq, p, grid, stream)
                            : launch_one<KIND, HEADS, 256, GATHER, false>(tk, tq, p, grid, stream);
}

template <int KIND, bool GATHER>
static cudaError_t launch_kind(const CUtensorMap& tk, const CUtensorMap& tq, const ScanParams& p,
                               int row_bytes, int grid, cudaStream_t stream) {
    switch (p.H) {
        case 4: return launch_heads<KIND, 4, GATHER>(tk, tq, p, row_bytes, grid, stream);
        case 8: return launch_heads<KIND, 8, GATHER>(tk, tq, p, row_bytes, grid, stream);
        case 16: return launch_heads<KIND, 16, GATHER>(tk, tq, p, row_bytes, grid, stream);
        case 32: return launch_heads<KIND, 32, GATHER>(tk, tq, p, row_bytes, grid, stream);
        case 64: return launch_heads<KIND, 64, GATHER>(tk, tq, p, row_bytes, grid, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <bool GATHER>
static cudaError_t launch_any(const CUtensorMap& tk, const CUtensorMap& tq, const ScanParams& p,
                              int grid, cudaStream_t stream) {
    if (p.nitems <= 0 || grid <= 0) return cudaSuccess;
    const int row_bytes = p.D * p.esize;
    switch (p.dtype) {
        case PIVOT_E4M3: return launch_kind<KIND_F8, GATHER>(tk, tq, p, row_bytes, grid, stream);
        case PIVOT_BF16: return launch_kind<KIND_F16, GATHER>(tk, tq, p, row_bytes, grid, stream);
        default: return cudaErrorInvalidValue;   // fp32 inputs are scored on the CUDA cores
    }
}

cudaError_t launch_scan_umma(const CUtensorMap& tk, const CUtensorMap& tq, const ScanParams& p,
                             int grid, cudaStream_t stream) {
    return launch_any<false>(tk, tq, p, grid, stream);
}

cudaError_t launch_refine_umma(const CUtensorMap& tmap_q, const ScanParams& p, int grid,
                               cudaStream_t stream) {
    // the key operand is gathered with cp.async from p.kbase; its tensor-map
    // slot is unused, so the query map fills it
    return launch_any<true>(tmap_q, tmap_q, p, grid, stream);
}

}  // namespace pivot
