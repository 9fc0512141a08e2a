// proxy_reuse.cu -- the proxy query of a group and PIVOT-Reuse.
//
// Proxy (abstract of arXiv 2607.24593: a group is aggregated into one proxy
// query; "PIVOT 설명 ... 10분 만에 구현하기", section "How It Works": the
// proxy is the mean of the group).  Per element, in fp32 and in member
// order, without fused multiply-add:
//     x_m = q value * q scale;   pq = (x_0 + x_1 + ... + x_{n-1}) / n
// and the same for the head weights; then stored in the input format (bf16
// round-to-nearest-even; e4m3 with one scale amax/448, saturating RNE).  A
// one-member group is copied unchanged.
//
// Reuse (same abstract): every member takes the proxy's top-k, i.e. the
// first k candidates in rank order, minus the positions after itself.
#include "common.cuh"
#include "kernels.h"

namespace pivot {

namespace {

constexpr int RED_THREADS = 256;

template <int DT>
__global__ void __launch_bounds__(RED_THREADS) proxy_reduce_kernel(const ReduceParams p) {
    extern __shared__ float qbar_s[];          // H*D (e4m3 only)
    __shared__ float red_s[RED_THREADS / 32];
    const int j = blockIdx.x;
    const size_t HD = (size_t)p.H * p.D;
    long long m0;
    int n;
    if (p.seg.tok) {   // packed group j of a ragged batch
        const SegGroup sg = seg_group(p.seg, p.g, j);
        m0 = sg.first;
        n = sg.n;
    } else {
        m0 = (long long)j * p.group_stride_members;
        n = (int)min((long long)p.g, (long long)p.nmembers_total - m0);
    }
    if (n <= 0) return;

    if (n == 1) {   // a group of one is its member
        const size_t esz = DT == PIVOT_F32 ? 4 : (DT == PIVOT_BF16 ? 2 : 1);
        const uint8_t* src = static_cast<const uint8_t*>(p.q) + (size_t)m0 * HD * esz;
        uint8_t* dst = static_cast<uint8_t*>(p.pq) + (size_t)j * HD * esz;
        for (size_t i = threadIdx.x; i < HD * esz; i += RED_THREADS) dst[i] = src[i];
        for (int h = threadIdx.x; h < p.H; h += RED_THREADS)
            p.pw[(size_t)j * p.H + h] = p.w[(size_t)m0 * p.H + h];
        if (DT == PIVOT_E4M3 && threadIdx.x == 0) p.pq_scale[j] = p.q_scale[m0];
        return;
    }

    const float fn = (float)n;
    float amax = 0.0f;
    // 16 bytes of a member row at a time (H*D*esize is a multiple of 16):
    // the same per-element sums, in member order, as one element at a time
    constexpr int ESZ = DT == PIVOT_F32 ? 4 : (DT == PIVOT_BF16 ? 2 : 1);
    constexpr int VE = 16 / ESZ;
    const size_t nchunks = HD / VE;
    const uint8_t* qb8 = static_cast<const uint8_t*>(p.q);
    for (size_t c = threadIdx.x; c < nchunks; c += RED_THREADS) {
        float acc[VE];
#pragma unroll 4
        for (int m = 0; m < n; ++m) {
            const size_t row = (size_t)(m0 + m);
            const uint4 raw = *reinterpret_cast<const uint4*>(qb8 + (row * HD + c * VE) * ESZ);
            const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
            float v[VE];
            if constexpr (DT == PIVOT_F32) {
#pragma unroll
                for (int e = 0; e < 4; ++e) v[e] = __uint_as_float(wd[e]);
            } else if constexpr (DT == PIVOT_BF16) {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    v[e] = bf16_to_f32((uint16_t)(wd[e >> 1] >> ((e & 1) * 16)));
            } else {
                const float sc = p.q_scale[row];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    v[e] = __fmul_rn(e4m3_to_f32((uint8_t)(wd[e >> 2] >> ((e & 3) * 8))), sc);
            }
#pragma unroll
            for (int e = 0; e < VE; ++e) acc[e] = m == 0 ? v[e] : __fadd_rn(acc[e], v[e]);
        }
        float qb[VE];
#pragma unroll
        for (int e = 0; e < VE; ++e) qb[e] = __fdiv_rn(acc[e], fn);
        if constexpr (DT == PIVOT_F32) {
            *reinterpret_cast<float4*>(static_cast<float*>(p.pq) + (size_t)j * HD + c * VE) =
                make_float4(qb[0], qb[1], qb[2], qb[3]);
        } else if constexpr (DT == PIVOT_BF16) {
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint16_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(qb[2 * e]));
                const uint16_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(qb[2 * e + 1]));
                o[e] = (uint32_t)lo | ((uint32_t)hi << 16);
            }
            *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.pq) + (size_t)j * HD + c * VE) =
                make_uint4(o[0], o[1], o[2], o[3]);
        } else {
#pragma unroll
            for (int e = 0; e < VE; ++e) {
                qbar_s[c * VE + e] = qb[e];
                amax = fmaxf(amax, fabsf(qb[e]));
            }
        }
    }
    for (int h = threadIdx.x; h < p.H; h += RED_THREADS) {
        float acc = p.w[(size_t)m0 * p.H + h];
        for (int m = 1; m < n; ++m) acc = __fadd_rn(acc, p.w[(size_t)(m0 + m) * p.H + h]);
        p.pw[(size_t)j * p.H + h] = __fdiv_rn(acc, fn);
    }
    if constexpr (DT == PIVOT_E4M3) {
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if ((threadIdx.x & 31) == 0) red_s[threadIdx.x >> 5] = amax;
        __syncthreads();
        float a = 0.0f;
        for (int w = 0; w < RED_THREADS / 32; ++w) a = fmaxf(a, red_s[w]);
        const float s = a > 0.0f ? __fdiv_rn(a, 448.0f) : 1.0f;
        uint8_t* dst = static_cast<uint8_t*>(p.pq) + (size_t)j * HD;
        for (size_t c = threadIdx.x; c < HD / 16; c += RED_THREADS) {
            uint32_t o[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int e = 0; e < 16; ++e)
                o[e >> 2] |= (uint32_t)f32_to_e4m3_satfinite(__fdiv_rn(qbar_s[c * 16 + e], s))
                             << ((e & 3) * 8);
            *reinterpret_cast<uint4*>(dst + c * 16) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        if (threadIdx.x == 0) p.pq_scale[j] = s;
    }
}

// One warp per member row: compact the first topk candidates to those <= lim.
__device__ __forceinline__ void reuse_row(const int32_t* c, int topk, int lim, int32_t* o) {
    const int lane = threadIdx.x & 31;
    int n = 0;
    for (int i0 = 0; i0 < topk; i0 += 32) {
        const int i = i0 + lane;
        const int32_t s = i < topk ? c[i] : -1;
        const bool ok = s >= 0 && s <= lim;
        const unsigned bal = __ballot_sync(0xffffffffu, ok);
        if (ok) o[n + __popc(bal & ((1u << lane) - 1u))] = s;
        n += __popc(bal);
    }
    for (int i = n + lane; i < topk; i += 32) o[i] = -1;
}

__global__ void reuse_kernel(int t_begin, int t_end, int g, const int32_t* cand, int C, int topk,
                             int32_t* idx, int lim_shift, int out_stride) {
    const int t = t_begin + blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (t >= t_end) return;
    const int j = t / g - t_begin / g;
    reuse_row(cand + (size_t)j * C, topk, t - lim_shift, idx + (size_t)(t - t_begin) * out_stride);
}

__global__ void reuse_varlen_kernel(const SegTable seg, int T, int g, const int32_t* cand, int C,
                                    int topk, int32_t* idx) {
    const int t = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (t >= T) return;
    const int b = seg_find(seg.tok, seg.nseq, t);
    const int j = seg.grp[b] + (t - seg.tok[b]) / g;
    reuse_row(cand + (size_t)j * C, topk, t - seg.tok[b], idx + (size_t)t * topk);
}

constexpr int WRITE_INTS_MAX = 960;   // 3840 bytes: under the 4 KB parameter limit
struct IntBlock {
    int32_t v[WRITE_INTS_MAX];
};

__global__ void write_ints_kernel(int32_t* dst, const IntBlock blk, int n) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) dst[i] = blk.v[i];
}

__global__ void decode_reuse_kernel(int B, int Gm, int maxlen, const int32_t* cache_len,
                                    const int32_t* cand, int C, int topk, int32_t* idx) {
    const int r = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (r >= B * Gm) return;
    const int b = r / Gm, m = r % Gm;
    const int n = cache_len[b];
    int lim = n - Gm + m;
    if (n < Gm || n > maxlen) {
        if ((threadIdx.x & 31) == 0) raise_error(ERRBIT_DATA);
        lim = -1;
    }
    reuse_row(cand + (size_t)b * C, topk, lim, idx + (size_t)r * topk);
}

// Window union ("Sparse Attention의 Indexer", Fig. 3, the window inside the
// candidates): an ascending row united with [a, t], a = max(0, t - window + 1),
// is its entries below a followed by a..t (entries in [a, t] are the window's
// own).  One warp per row.
__global__ void window_union_kernel(const int32_t* idx, int rows, int k, int t_begin,
                                    const int32_t* positions, int window, int32_t* out,
                                    int in_stride) {
    const int r = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (r >= rows) return;
    const int lane = threadIdx.x & 31;
    const int t = positions ? positions[r] : t_begin + r;
    const int a = t - window + 1 > 0 ? t - window + 1 : 0;
    // in place (out == idx, in_stride == k + window) every read of a chunk
    // precedes its writes, which never pass the entries read
    const int32_t* in = idx + (size_t)r * in_stride;
    int32_t* o = out + (size_t)r * (k + window);
    int n = 0;
    for (int i0 = 0; i0 < k; i0 += 32) {
        const int i = i0 + lane;
        const int32_t s = i < k ? in[i] : -1;
        const bool keep = s >= 0 && s < a;
        const unsigned bal = __ballot_sync(0xffffffffu, keep);
        if (keep) o[n + __popc(bal & ((1u << lane) - 1u))] = s;
        n += __popc(bal);
    }
    const int nw = t >= a ? t - a + 1 : 0;   // t < 0 (no position) leaves the window empty
    for (int i = lane; i < nw; i += 32) o[n + i] = a + i;
    for (int i = n + nw + lane; i < k + window; i += 32) o[i] = -1;
}

}  // namespace

namespace {

// One thread a group: the rank-ordered scores fall along the row (-inf
// padding last), so the count is one binary search for the last score at
// or above rho times the k-th.
__global__ void adaptive_count_kernel(const float* cs, int G, int C, int topk, float rho,
                                      int32_t* count) {
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= G) return;
    const float* row = cs + (size_t)j * C;
    int valid = 0, hi = C;   // valid = entries with a finite score
    while (valid < hi) {
        const int mid = (valid + hi) >> 1;
        if (row[mid] > -INFINITY) valid = mid + 1;
        else hi = mid;
    }
    const int kk = topk < valid ? topk : valid;
    int n = C;
    if (kk > 0 && row[kk - 1] > 0.0f) {
        const float T = rho * row[kk - 1];
        int lo = kk;
        hi = valid;
        while (lo < hi) {   // the first entry below T, from the k-th on
            const int mid = (lo + hi) >> 1;
            if (row[mid] >= T) lo = mid + 1;
            else hi = mid;
        }
        n = lo;
    }
    count[j] = n < kk ? kk : n;
}

}  // namespace

cudaError_t launch_adaptive_count(const float* cand_score, int G, int C, int topk, float rho,
                                  int32_t* count, cudaStream_t stream) {
    if (G <= 0) return cudaSuccess;
    adaptive_count_kernel<<<ceil_div(G, 256), 256, 0, stream>>>(cand_score, G, C, topk, rho, count);
    return cudaGetLastError();
}

cudaError_t launch_window_union(const int32_t* idx, int rows, int k, int t_begin,
                                const int32_t* positions, int window, int32_t* out,
                                cudaStream_t stream, int in_stride) {
    if (rows <= 0) return cudaSuccess;
    const int wpb = 8;
    window_union_kernel<<<ceil_div(rows, wpb), wpb * 32, 0, stream>>>(
        idx, rows, k, t_begin, positions, window, out, in_stride ? in_stride : k);
    return cudaGetLastError();
}

cudaError_t launch_proxy_reduce(const ReduceParams& p, cudaStream_t stream) {
    if (p.ngroups <= 0) return cudaSuccess;
    const size_t smem = p.dtype == PIVOT_E4M3 ? (size_t)p.H * p.D * 4 : 0;
    switch (p.dtype) {
        case PIVOT_F32:
            proxy_reduce_kernel<PIVOT_F32><<<p.ngroups, RED_THREADS, 0, stream>>>(p);
            break;
        case PIVOT_BF16:
            proxy_reduce_kernel<PIVOT_BF16><<<p.ngroups, RED_THREADS, 0, stream>>>(p);
            break;
        default: {
            cudaError_t e = cudaFuncSetAttribute(proxy_reduce_kernel<PIVOT_E4M3>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem);
            if (e != cudaSuccess) return e;
            proxy_reduce_kernel<PIVOT_E4M3><<<p.ngroups, RED_THREADS, smem, stream>>>(p);
        }
    }
    return cudaGetLastError();
}

cudaError_t launch_reuse(int t_begin, int t_end, int g, const int32_t* cand, int C, int topk,
                         int32_t* idx, cudaStream_t stream, int lim_shift, int out_stride) {
    const int rows = t_end - t_begin;
    if (rows <= 0) return cudaSuccess;
    const int wpb = 8;
    reuse_kernel<<<ceil_div(rows, wpb), wpb * 32, 0, stream>>>(
        t_begin, t_end, g, cand, C, topk, idx, lim_shift, out_stride ? out_stride : topk);
    return cudaGetLastError();
}

cudaError_t launch_reuse_varlen(const SegTable& seg, int T, int g, const int32_t* cand, int C,
                                int topk, int32_t* idx, cudaStream_t stream) {
    if (T <= 0) return cudaSuccess;
    const int wpb = 8;
    reuse_varlen_kernel<<<ceil_div(T, wpb), wpb * 32, 0, stream>>>(seg, T, g, cand, C, topk, idx);
    return cudaGetLastError();
}

cudaError_t launch_write_ints(int32_t* dst, const int32_t* host, int n, cudaStream_t stream) {
    if (n < 0 || n > WRITE_INTS_MAX) return cudaErrorInvalidValue;
    if (n == 0) return cudaSuccess;
    IntBlock blk;
    for (int i = 0; i < n; ++i) blk.v[i] = host[i];
    write_ints_kernel<<<1, 256, 0, stream>>>(dst, blk, n);
    return cudaGetLastError();
}

cudaError_t launch_decode_reuse(int B, int Gm, int maxlen, const int32_t* cache_len,
                                const int32_t* cand, int C, int topk, int32_t* idx,
                                cudaStream_t stream) {
    const int rows = B * Gm;
    if (rows <= 0) return cudaSuccess;
    const int wpb = 8;
    decode_reuse_kernel<<<ceil_div(rows, wpb), wpb * 32, 0, stream>>>(B, Gm, maxlen, cache_len,
                                                                       cand, C, topk, idx);
    return cudaGetLastError();
}

}  // namespace pivot
