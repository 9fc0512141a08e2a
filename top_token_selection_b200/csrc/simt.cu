// simt.cu -- indexer scores on the CUDA cores.
//
// Two users: PIVOT-Refine's re-scoring of each group's candidate keys
// (abstract of arXiv 2607.24593: each member re-scores the candidate set with
// its own indexer), where the keys are gathered by candidate index; and the
// scan for shapes the tensor-core tiling does not cover (H not dividing 256,
// or a key row that is not 128 or 256 bytes).
//
// A CTA takes 128 keys (one per thread), stages them transposed in shared
// memory as fp32, then walks its query rows: each row's H*D query values
// and H weights are staged in shared memory and every thread computes
//     I(r, s) = (sum_h w[r,h] * max(0, sum_d q[r,h,d] * k[s,d])) * q_scale * k_scale.
#include "common.cuh"
#include "kernels.h"

namespace pivot {

namespace {

constexpr int ST = 128;   // keys per CTA

__device__ __forceinline__ float load_elem(int dtype, const void* base, size_t i) {
    if (dtype == PIVOT_F32) return static_cast<const float*>(base)[i];
    if (dtype == PIVOT_BF16) return bf16_to_f32(static_cast<const uint16_t*>(base)[i]);
    return e4m3_to_f32(static_cast<const uint8_t*>(base)[i]);
}

__device__ __forceinline__ int lim_of(int kind, int r, int L, int g, int Gm, int maxlen,
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

// Score rows [r_first, r_first + rows) against the 128 keys staged in kT.
__device__ void score_rows(int dtype, int H, int D, const void* q, const float* q_scale,
                           const float* w, int qrow_base, int r_first, int rows,
                           const float* kT, float* qs, float* ws, float sk, int s_pos,
                           bool key_ok, int kind, int L, int g, int Gm, int maxlen,
                           const int32_t* cache_len, float* S, long long S_stride, int row0,
                           int col) {
    const size_t HD = (size_t)H * D;
    for (int pr = 0; pr < rows; ++pr) {
        const int r = r_first + pr;
        const size_t qr = (size_t)(r - qrow_base);
        __syncthreads();
        for (size_t i = threadIdx.x; i < HD; i += ST) qs[i] = load_elem(dtype, q, qr * HD + i);
        for (int h = threadIdx.x; h < H; h += ST) ws[h] = w[qr * H + h];
        __syncthreads();
        bool ok;
        const int lim = lim_of(kind, r, L, g, Gm, maxlen, cache_len, ok);
        float acc = 0.0f;
        for (int h = 0; h < H; ++h) {
            float dot = 0.0f;
            for (int d = 0; d < D; ++d) dot = fmaf(qs[h * D + d], kT[d * ST + threadIdx.x], dot);
            acc = fmaf(ws[h], fmaxf(dot, 0.0f), acc);
        }
        const float sq = q_scale ? q_scale[qr] : 1.0f;
        if (key_ok && ok && s_pos <= lim)
            S[(size_t)(r - row0) * S_stride + col] = acc * sq * sk;
    }
}

__global__ void __launch_bounds__(ST) scan_simt_kernel(const void* q, const void* k,
                                                       const ScanParams p) {
    extern __shared__ float sm[];
    float* kT = sm;                        // D * 128
    float* qs = kT + p.D * ST;             // H * D
    float* ws = qs + (size_t)p.H * p.D;    // H
    const int blk = blockIdx.x / p.items_per_block;
    const int tile = blockIdx.x % p.items_per_block;
    const int r_first = p.row0 + blk * p.P;
    const int rows = min(p.P, p.row0 + p.nrows - r_first);
    bool ok;
    const int maxlim = lim_of(p.kind, r_first + rows - 1, p.L, p.g, p.Gm, p.maxlen, p.cache_len, ok);
    if (!ok || tile * ST > maxlim) return;
    int keybase = 0;
    if (p.kind == SCAN_DECODE_DENSE) keybase = (r_first / p.Gm) * p.maxlen;
    if (p.kind == SCAN_DECODE_PROXY) keybase = r_first * p.maxlen;
    const int s = tile * ST + threadIdx.x;
    const bool key_ok = s <= maxlim;
    for (int d = 0; d < p.D; ++d)
        kT[d * ST + threadIdx.x] =
            key_ok ? load_elem(p.dtype, k, (size_t)(keybase + s) * p.D + d) : 0.0f;
    const float sk = (p.k_scale && key_ok) ? p.k_scale[keybase + s] : 1.0f;
    score_rows(p.dtype, p.H, p.D, q, p.q_scale, p.w, p.qrow_base, r_first, rows, kT, qs, ws, sk,
               s, key_ok, p.kind, p.L, p.g, p.Gm, p.maxlen, p.cache_len, p.S, p.S_stride, p.row0,
               s);
}

__global__ void __launch_bounds__(ST) refine_simt_kernel(const RefineParams p) {
    extern __shared__ float sm[];
    float* kT = sm;
    float* qs = kT + p.D * ST;
    float* ws = qs + (size_t)p.H * p.D;
    const int ntiles = ceil_div(p.C, ST);
    const int gi = blockIdx.x / ntiles;            // group of this CTA (relative)
    const int tile = blockIdx.x % ntiles;
    const int grp = p.cand_base + gi;
    const int gsize = (p.kind == SCAN_DECODE_DENSE) ? p.Gm : p.g;
    int r_first = grp * gsize;
    int r_last = r_first + gsize;                  // exclusive
    if (r_first < p.row0) r_first = p.row0;
    if (r_last > p.row0 + p.nrows) r_last = p.row0 + p.nrows;
    if (r_first >= r_last) return;
    const int c = tile * ST + threadIdx.x;
    int keyrow = -1;
    int pos = -1;
    if (c < p.C) {
        pos = p.cand[(size_t)gi * p.C + c];
        int nkeys = p.L;
        int base = 0;
        if (p.kind == SCAN_DECODE_DENSE) { nkeys = p.maxlen; base = grp * p.maxlen; }
        if (pos >= 0 && pos < nkeys) keyrow = base + pos;
    }
    const bool key_ok = keyrow >= 0;
    for (int d = 0; d < p.D; ++d)
        kT[d * ST + threadIdx.x] = key_ok ? load_elem(p.dtype, p.k, (size_t)keyrow * p.D + d) : 0.0f;
    // Refine scores are stored without the key scale: the candidate
    // selection multiplies it in, in the same order ((acc * sq) * sk).
    (void)keyrow;
    const float sk = 1.0f;
    score_rows(p.dtype, p.H, p.D, p.q, p.q_scale, p.w, p.qrow_base, r_first, r_last - r_first, kT,
               qs, ws, sk, key_ok ? pos : 0x7fffffff, key_ok && c < p.C, p.kind, p.L, p.g, p.Gm,
               p.maxlen, p.cache_len, p.S, p.C, p.row0, c);
}

}  // namespace

cudaError_t launch_scan_simt(const void* q, const void* k, const ScanParams& p,
                             cudaStream_t stream) {
    if (p.nrows <= 0) return cudaSuccess;
    const int nblocks = ceil_div(p.nrows, p.P);
    const size_t smem = ((size_t)p.D * ST + (size_t)p.H * p.D + p.H) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(scan_simt_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // items_per_block = key tiles covering the longest prefix of the launch
    scan_simt_kernel<<<nblocks * p.items_per_block, ST, smem, stream>>>(q, k, p);
    return cudaGetLastError();
}

cudaError_t launch_refine_simt(const RefineParams& p, cudaStream_t stream) {
    if (p.nrows <= 0) return cudaSuccess;
    const int gsize = (p.kind == SCAN_DECODE_DENSE) ? p.Gm : p.g;
    const int g_first = p.cand_base;
    const int g_last = (p.row0 + p.nrows - 1) / gsize;
    const int ngroups = g_last - g_first + 1;
    const size_t smem = ((size_t)p.D * ST + (size_t)p.H * p.D + p.H) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(refine_simt_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    refine_simt_kernel<<<ngroups * ceil_div(p.C, ST), ST, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace pivot
