// C entry points over the host-emulated csrc/simt.cu (the CUDA-core scan and
// Refine scoring for shapes outside the tensor-core tiling), for
// tests/test_simt_emu_cpu.py: each call fills the kernel's parameter block as
// the library does and runs its launcher.
#include <cstdint>

#include "kernels.h"
#include "pivot.h"

namespace pivot {
uint32_t g_error_word = 0;
}
using namespace pivot;

extern "C" {

uint32_t emu_error_word() {
    const uint32_t w = g_error_word;
    g_error_word = 0;
    return w;
}

// Rows [row0, row0 + nrows) of `kind` into S (row r at S + (r - row0) * stride),
// in blocks of P rows, key tiles covering [0, maxlim_total].
int emu_scan_simt(int kind, int dtype, int H, int D, int P, const void* q, const float* q_scale,
                  const float* w, const void* k, const float* k_scale, int L, int g, int Gm,
                  int maxlen, const int32_t* cache_len, int row0, int nrows, int qrow_base,
                  int maxlim_total, float* S, long long stride) {
    ScanParams p{};
    p.kind = kind;
    p.dtype = dtype;
    p.esize = dtype == PIVOT_F32 ? 4 : (dtype == PIVOT_BF16 ? 2 : 1);
    p.H = H;
    p.D = D;
    p.P = P;
    p.row0 = row0;
    p.nrows = nrows;
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
    p.tiles_per_item = 1;
    p.items_per_block = (maxlim_total + 1 + 127) / 128;
    p.nitems = ((nrows + P - 1) / P) * p.items_per_block;
    return launch_scan_simt(q, k, p, nullptr);
}

int emu_refine_simt(int kind, int dtype, int H, int D, const void* q, const float* q_scale,
                    const float* w, const void* k, int L, int g, int Gm, int maxlen,
                    const int32_t* cache_len, const int32_t* cand, int cand_base, int C, int row0,
                    int nrows, float* S) {
    RefineParams p{};
    p.dtype = dtype;
    p.esize = dtype == PIVOT_F32 ? 4 : (dtype == PIVOT_BF16 ? 2 : 1);
    p.H = H;
    p.D = D;
    p.kind = kind;
    p.row0 = row0;
    p.nrows = nrows;
    p.qrow_base = 0;
    p.L = L;
    p.g = g;
    p.Gm = Gm;
    p.maxlen = maxlen;
    p.cache_len = cache_len;
    p.q = q;
    p.q_scale = q_scale;
    p.w = w;
    p.k = k;
    p.cand = cand;
    p.cand_base = cand_base;
    p.C = C;
    p.S = S;
    return launch_refine_simt(p, nullptr);
}

}  // extern "C"
