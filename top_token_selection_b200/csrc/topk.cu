// topk.cu -- exact per-row top-K selection with the indexer's tie-break.
//
// The indexer returns positions only, the k highest scores of the row
// ("Sparse Attention의 Indexer", Fig. 1: top-k keeps the k largest selection
// scores).  Order: higher score first, equal scores by lower position, -0
// equal to +0.  Each entry gets a 64-bit key
//     key = ordered(score) << 32 | (0xFFFFFFFF - position)
// which is unique per row, so "the K largest keys" is exactly the answer.
//
// One CTA per row:
//   1. histogram of the top 12 key bits over the row (warp-aggregated
//      shared-memory atomics);
//   2. the bin B holding the K-th largest; entries of higher bins are in;
//   3. entries of bin B go to a shared-memory boundary buffer (or, if it
//      overflows, are re-read from global memory), where an 8-bit-digit
//      radix select over the remaining 52 key bits picks the exact rest;
//   4. the K winners are sorted in shared memory (bitonic) and written.
#include "common.cuh"
#include "kernels.h"

namespace pivot {

namespace {

constexpr int SEL_THREADS = 512;
constexpr int HIST_BINS = 4096;     // top 12 bits of the ordered score

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

struct RowView {
    const float* S;
    const int32_t* cand;   // null: position = entry index
    int n;                 // entries
    int lim;               // valid positions are <= lim
};

// Key of entry i, or 0 when the entry is not eligible.
__device__ __forceinline__ uint64_t entry_key(const RowView& v, int i) {
    int pos = i;
    if (v.cand) {
        pos = v.cand[i];
        if (pos < 0 || pos > v.lim) return 0;
    }
    const uint32_t u = ordered_key(v.S[i]);
    return ((uint64_t)u << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)pos);
}

__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool active) {
    const unsigned mask = __ballot_sync(0xffffffffu, active);
    if (!active) return;
    const unsigned peers = __match_any_sync(mask, bin);
    const int leader = __ffs(peers) - 1;
    if ((threadIdx.x & 31) == leader) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
}

// Block-wide: find the largest bin b with sum_{bins >= b} hist >= need, over
// `nbins` bins.  Returns b and the count strictly above it in *above.
// Requires nbins % SEL_THREADS == 0 or nbins <= SEL_THREADS.
__device__ int find_threshold_bin(const uint32_t* hist, int nbins, uint32_t need,
                                  uint32_t* scratch, uint32_t* above) {
    __shared__ int s_bin;
    __shared__ uint32_t s_above;
    const int per = nbins >= SEL_THREADS ? nbins / SEL_THREADS : 1;
    const int t = threadIdx.x;
    // thread t owns bins [nbins - (t+1)*per, nbins - t*per) (descending order)
    uint32_t local = 0;
    const int hi = nbins - t * per;        // exclusive
    const int lo = hi - per;
    if (lo >= 0)
        for (int b = lo; b < hi; ++b) local += hist[b];
    // inclusive scan over threads (descending bins)
    const int lane = t & 31, wid = t >> 5;
    uint32_t x = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[wid] = x;
    if (t == 0) { s_bin = -1; s_above = 0; }
    __syncthreads();
    if (wid == 0) {
        uint32_t w = lane < SEL_THREADS / 32 ? scratch[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < SEL_THREADS / 32) scratch[32 + lane] = w;   // inclusive warp totals
    }
    __syncthreads();
    const uint32_t before = (wid > 0 ? scratch[32 + wid - 1] : 0) + x - local;  // exclusive
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
    return s_bin;
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

__global__ void __launch_bounds__(SEL_THREADS)
    select_kernel(const SelectParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem);                   // HIST_BINS
    uint32_t* scratch = hist + HIST_BINS;                                  // 64
    uint64_t* sel = reinterpret_cast<uint64_t*>(scratch + 64);             // pow2(K)
    int M2 = 1;
    while (M2 < p.K) M2 <<= 1;
    uint64_t* tail = sel + M2;                                             // tail_cap
    __shared__ uint32_t s_nsel, s_ntail;

    const int r = p.row0 + blockIdx.x;
    int32_t* out = p.out_idx + (size_t)(r - p.out_base) * p.K;
    float* outs = p.out_score ? p.out_score + (size_t)(r - p.out_base) * p.K : nullptr;

    bool ok;
    const int lim = row_limit(p.scan_kind, r, p.L, p.g, p.Gm, p.maxlen, p.cache_len, ok);
    RowView v;
    v.S = p.S + (size_t)(r - p.row0) * p.S_stride;
    v.lim = lim;
    if (p.kind == SEL_PREFIX) {
        v.cand = nullptr;
        v.n = ok ? lim + 1 : 0;
    } else {
        const int grp = (p.scan_kind == SCAN_DECODE_DENSE) ? r / p.Gm : r / p.g;
        v.cand = p.cand + (size_t)(grp - p.cand_base) * p.C;
        v.n = ok ? p.C : 0;
    }
    if (!ok && threadIdx.x == 0) raise_error(ERRBIT_DATA);

    // 1. histogram of the top 12 bits
    for (int b = threadIdx.x; b < HIST_BINS; b += SEL_THREADS) hist[b] = 0;
    if (threadIdx.x == 0) { s_nsel = 0; s_ntail = 0; }
    __syncthreads();
    const bool vec = (v.cand == nullptr) && ((reinterpret_cast<uintptr_t>(v.S) & 15) == 0);
    if (vec) {
        const int n4 = v.n / 4;
        const float4* S4 = reinterpret_cast<const float4*>(v.S);
        for (int i0 = 0; i0 < n4; i0 += SEL_THREADS) {
            const int i = i0 + threadIdx.x;
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < n4) x = S4[i];
            const bool a = i < n4;
            hist_add(hist, ordered_key(x.x) >> 20, a);
            hist_add(hist, ordered_key(x.y) >> 20, a);
            hist_add(hist, ordered_key(x.z) >> 20, a);
            hist_add(hist, ordered_key(x.w) >> 20, a);
        }
        const int i = n4 * 4 + threadIdx.x;
        const bool a = i < v.n;
        hist_add(hist, a ? ordered_key(v.S[i]) >> 20 : 0u, a);
    } else {
        for (int i0 = 0; i0 < v.n; i0 += SEL_THREADS) {
            const int i = i0 + threadIdx.x;
            uint64_t k = i < v.n ? entry_key(v, i) : 0;
            hist_add(hist, (uint32_t)(k >> 52), k != 0);
        }
    }
    __syncthreads();

    // total eligible
    uint32_t total_local = 0;
    for (int b = threadIdx.x; b < HIST_BINS; b += SEL_THREADS) total_local += hist[b];
    for (int o = 16; o > 0; o >>= 1) total_local += __shfl_xor_sync(0xffffffffu, total_local, o);
    if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = total_local;
    __syncthreads();
    uint32_t total = 0;
    for (int w = 0; w < SEL_THREADS / 32; ++w) total += scratch[w];
    __syncthreads();
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
            sel[atomicAdd(&s_nsel, 1u)] = k;
        } else if (b == bin) {
            const uint32_t slot = atomicAdd(&s_ntail, 1u);
            if (slot < (uint32_t)p.tail_cap) tail[slot] = k;
        }
    }
    __syncthreads();

    // 4. resolve the boundary bin
    if (bin >= 0 && need > 0) {
        const uint32_t ntail = s_ntail;
        uint64_t mask, prefix;
        if (ntail == need) {
            mask = 0; prefix = 0;   // take all of them
        } else if (ntail <= (uint32_t)p.tail_cap) {
            radix_select_tail<true>(v, tail, (int)ntail, (uint32_t)bin, need, hist, scratch,
                                    &mask, &prefix);
        } else {
            radix_select_tail<false>(v, nullptr, 0, (uint32_t)bin, need, hist, scratch, &mask,
                                     &prefix);
        }
        if (ntail <= (uint32_t)p.tail_cap) {
            for (uint32_t i = threadIdx.x; i < ntail; i += SEL_THREADS) {
                const uint64_t k = tail[i];
                if ((k & mask) >= prefix) sel[atomicAdd(&s_nsel, 1u)] = k;
            }
        } else {
            for (int i = threadIdx.x; i < v.n; i += SEL_THREADS) {
                const uint64_t k = entry_key(v, i);
                if (k != 0 && (int)(k >> 52) == bin && (k & mask) >= prefix)
                    sel[atomicAdd(&s_nsel, 1u)] = k;
            }
        }
        __syncthreads();
    }

    // 5. rank order: bitonic sort, descending, over the next power of two
    int M = 1;
    while ((uint32_t)M < Kp) M <<= 1;
    for (int i = Kp + threadIdx.x; i < M; i += SEL_THREADS) sel[i] = 0;
    __syncthreads();
    for (int kk = 2; kk <= M; kk <<= 1) {
        for (int j = kk >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < M; i += SEL_THREADS) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const uint64_t a = sel[i], b = sel[ixj];
                    const bool desc = (i & kk) == 0;
                    if (desc ? (a < b) : (a > b)) {
                        sel[i] = b;
                        sel[ixj] = a;
                    }
                }
            }
            __syncthreads();
        }
    }

    // 6. write
    for (int i = threadIdx.x; i < p.K; i += SEL_THREADS) {
        if ((uint32_t)i < Kp) {
            const uint64_t k = sel[i];
            out[i] = (int32_t)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFu));
            if (outs) outs[i] = key_to_float((uint32_t)(k >> 32));
        } else {
            out[i] = -1;
            if (outs) outs[i] = -INFINITY;
        }
    }
}

}  // namespace

size_t select_smem_bytes(int K, int tail_cap) {
    size_t m2 = 1;
    while (m2 < (size_t)K) m2 <<= 1;
    return HIST_BINS * 4 + 64 * 4 + m2 * 8 + (size_t)tail_cap * 8;
}

cudaError_t launch_select(const SelectParams& p, cudaStream_t stream) {
    if (p.nrows <= 0) return cudaSuccess;
    const size_t smem = select_smem_bytes(p.K, p.tail_cap);
    cudaError_t e =
        cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    select_kernel<<<p.nrows, SEL_THREADS, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace pivot
