// scan_umma.cu -- indexer scores on the 5th-generation tensor cores.
//
// Computes, for a block of P query rows (queries, or proxy queries) that
// share one key sequence, the indexer score of every key of the causal
// prefix:
//     I(r, s) = sum_h w[r,h] * ReLU(q[r,h] . k[s])      (x q_scale * k_scale)
// (dense indexer of "Sparse Attention의 Indexer", Fig. 1-2, in the multi-head
// form; the same scan serves the PIVOT proxy scan of the abstract of arXiv
// 2607.24593, run once per group with the proxy as the query).
//
// Mapping: keys on the MMA M axis (128 TMEM lanes), the P*H query heads on
// N (<= 256 columns).  Each epilogue thread owns one key and reduces its
// lane's columns over heads in registers -- no shuffles.  The query block is
// loaded once per work item and stays in shared memory; key tiles stream
// through a TMA ring.  Accumulators are double-buffered in TMEM (2 x 256
// columns) so the epilogue of tile i overlaps the MMAs of tile i+1.
//
// Warp roles (192 threads): warp 0 issues TMA, warp 1 allocates TMEM and
// issues tcgen05.mma, warps 2-5 run the epilogue.
#include "common.cuh"
#include "kernels.h"

namespace pivot {

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
    int blk, rows, row_first, t0, t1, keybase, maxlim;
    bool valid;
};

// Work item i = (row block, chunk of key tiles).  Items whose chunk starts
// beyond the block's causal extent are empty.  Every role walks the same
// item sequence.
__device__ __forceinline__ ItemInfo scan_item(const ScanParams& p, int item) {
    ItemInfo it;
    it.blk = item / p.items_per_block;
    int chunk = item % p.items_per_block;
    it.row_first = p.row0 + it.blk * p.P;
    int rows = p.row0 + p.nrows - it.row_first;
    it.rows = rows < p.P ? rows : p.P;
    bool ok;
    int maxlim = scan_row_lim(p, it.row_first + it.rows - 1, ok);
    it.maxlim = ok ? maxlim : -1;
    it.keybase = scan_key_base(p, it.row_first);
    int nt = ok ? (maxlim + 1 + 127) / 128 : 0;
    it.t0 = chunk * p.tiles_per_item;
    it.t1 = it.t0 + p.tiles_per_item < nt ? it.t0 + p.tiles_per_item : nt;
    it.valid = it.t0 < nt;
    return it;
}

template <int KIND, int HEADS, int ROWB>
__global__ void __launch_bounds__(192, 1)
    scan_umma_kernel(const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_q, const ScanParams p) {
    constexpr int KBLK = ROWB / 128;           // 128-byte K blocks per row
    constexpr int KSTEPS = ROWB / 32;          // one MMA consumes 32 bytes of K
    constexpr int A_BYTES = 128 * ROWB;        // one key tile
    constexpr int B_SLOT = 256 * ROWB;         // query block, N <= 256 rows
    constexpr int STAGES = ROWB == 128 ? 6 : 3;
    constexpr int PMAX = 256 / HEADS;
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
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    float* w_s = reinterpret_cast<float*>(tmem_holder + 4);   // [256]
    float* sq_s = w_s + 256;                                   // [PMAX]
    int* lim_s = reinterpret_cast<int*>(sq_s + PMAX);          // [PMAX]

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int N = p.P * HEADS;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bfull[i], 1);
            mbar_init(&bempty[i], 1);
            mbar_init(&accfull[i], 1);
            mbar_init(&accempty[i], 4);   // one arrive per epilogue warp
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

    if (warp == 0) {
        // ------------------------------------------------------------ TMA
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int nit = 0;
            // parity of the last load issued per stage / query slot (-1: none),
            // so every load can be waited for before the CTA exits
            int last_a[STAGES], last_b[2] = {-1, -1};
            for (int i = 0; i < STAGES; ++i) last_a[i] = -1;
            bool aborted = false;
            for (int item = blockIdx.x; item < p.nitems && !aborted; item += gridDim.x) {
                ItemInfo it = scan_item(p, item);
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
                    for (int kb = 0; kb < KBLK; ++kb)
                        tma_load_2d(sA + stage * A_BYTES + kb * (128 * 128), &tmap_k,
                                    &full[stage], kb * (128 / p.esize), it.keybase + t * 128);
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
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            const uint32_t idesc = make_idesc(FMT, 128, (uint32_t)N);
            int stage = 0;
            uint32_t phase = 0;
            int nit = 0, ntile = 0;
            bool aborted = false;
            for (int item = blockIdx.x; item < p.nitems && !aborted; item += gridDim.x) {
                ItemInfo it = scan_item(p, item);
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
    } else {
        // ------------------------------------------------------- epilogue
        const int ew = warp - 2;                  // 0..3
        const int quarter = warp & 3;             // TMEM lane quarter of this warp
        const int key_in_tile = quarter * 32 + lane;
        const int et = ew * 32 + lane;            // 0..127
        int ntile = 0;
        // Once a wait runs out the warp stops touching TMEM and memory but
        // keeps walking the items, so the named barriers shared by the four
        // epilogue warps are always reached.
        bool aborted = false;
        for (int item = blockIdx.x; item < p.nitems; item += gridDim.x) {
            ItemInfo it = scan_item(p, item);
            if (!it.valid) continue;
            named_bar_sync(1, 128);
            for (int i = et; i < N; i += 128) {
                const int pr = i / HEADS;
                w_s[i] = pr < it.rows
                             ? p.w[(size_t)(it.row_first + pr - p.qrow_base) * HEADS + i % HEADS]
                             : 0.0f;
            }
            for (int pr = et; pr < p.P; pr += 128) {
                bool ok = true;
                int lim = pr < it.rows ? scan_row_lim(p, it.row_first + pr, ok) : -1;
                lim_s[pr] = ok ? lim : -1;
                sq_s[pr] = (p.q_scale && pr < it.rows)
                               ? p.q_scale[it.row_first + pr - p.qrow_base]
                               : 1.0f;
            }
            named_bar_sync(1, 128);
            for (int t = it.t0; t < it.t1; ++t) {
                const int acc = ntile & 1;
                const uint32_t aph = (ntile >> 1) & 1;
                ++ntile;
                if (aborted) continue;
                const bool got = mbar_wait(&accfull[acc], aph);
                if (!__all_sync(0xffffffffu, got)) { aborted = true; continue; }
                tc_fence_after();
                const int s = t * 128 + key_in_tile;                 // key position
                const float sk =
                    (p.k_scale && s <= it.maxlim) ? p.k_scale[it.keybase + s] : 1.0f;
                const uint32_t taddr =
                    tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * 256);
                float rowacc = 0.0f;
                float v[32];
#pragma unroll 1
                for (int c0 = 0; c0 < N; c0 += 32) {
                    tmem_ld32(taddr + c0, v);
                    tmem_ld_wait();
                    if constexpr (HEADS <= 32) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            rowacc = fmaf(w_s[c0 + i], fmaxf(v[i], 0.0f), rowacc);
                            if ((i + 1) % HEADS == 0) {
                                const int pr = (c0 + i) / HEADS;
                                if (s <= lim_s[pr])
                                    p.S[(size_t)(it.row_first + pr - p.row0) * p.S_stride + s] =
                                        rowacc * sq_s[pr] * sk;
                                rowacc = 0.0f;
                            }
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            rowacc = fmaf(w_s[c0 + i], fmaxf(v[i], 0.0f), rowacc);
                        if ((c0 + 32) % HEADS == 0) {
                            const int pr = c0 / HEADS;
                            if (s <= lim_s[pr])
                                p.S[(size_t)(it.row_first + pr - p.row0) * p.S_stride + s] =
                                    rowacc * sq_s[pr] * sk;
                            rowacc = 0.0f;
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&accempty[acc]);
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

template <int KIND, int HEADS>
static cudaError_t launch_scan_heads(const CUtensorMap& tk, const CUtensorMap& tq,
                                     const ScanParams& p, int row_bytes, int grid,
                                     cudaStream_t stream) {
    if (row_bytes == 128) {
        auto kfn = scan_umma_kernel<KIND, HEADS, 128>;
        const int smem = scan_smem_bytes(128);
        cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        kfn<<<grid, 192, smem, stream>>>(tk, tq, p);
    } else {
        auto kfn = scan_umma_kernel<KIND, HEADS, 256>;
        const int smem = scan_smem_bytes(256);
        cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        kfn<<<grid, 192, smem, stream>>>(tk, tq, p);
    }
    return cudaGetLastError();
}

int scan_smem_bytes(int row_bytes) {
    const int stages = row_bytes == 128 ? 6 : 3;
    const int pmax = 64;
    return 1024 /*align slack*/ + 2 * 256 * row_bytes + stages * 128 * row_bytes +
           (2 * stages + 9) * 8 + 16 + 256 * 4 + pmax * 8;
}

template <int KIND>
static cudaError_t launch_scan_kind(const CUtensorMap& tk, const CUtensorMap& tq,
                                    const ScanParams& p, int row_bytes, int grid,
                                    cudaStream_t stream) {
    switch (p.H) {
        case 4: return launch_scan_heads<KIND, 4>(tk, tq, p, row_bytes, grid, stream);
        case 8: return launch_scan_heads<KIND, 8>(tk, tq, p, row_bytes, grid, stream);
        case 16: return launch_scan_heads<KIND, 16>(tk, tq, p, row_bytes, grid, stream);
        case 32: return launch_scan_heads<KIND, 32>(tk, tq, p, row_bytes, grid, stream);
        case 64: return launch_scan_heads<KIND, 64>(tk, tq, p, row_bytes, grid, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_scan_umma(const CUtensorMap& tk, const CUtensorMap& tq, const ScanParams& p,
                             int grid, cudaStream_t stream) {
    if (p.nitems <= 0 || grid <= 0) return cudaSuccess;
    const int row_bytes = p.D * p.esize;
    switch (p.dtype) {
        case PIVOT_E4M3: return launch_scan_kind<KIND_F8>(tk, tq, p, row_bytes, grid, stream);
        case PIVOT_BF16: return launch_scan_kind<KIND_F16>(tk, tq, p, row_bytes, grid, stream);
        default: return launch_scan_kind<KIND_TF32>(tk, tq, p, row_bytes, grid, stream);
    }
}

}  // namespace pivot
