// C entry points over the host-emulated csrc/proxy_reuse.cu, for
// tests/test_reuse_emu_cpu.py (ctypes): each call runs the library's own
// launcher, whose kernel launches run block by block on host threads.
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

int emu_reuse(int t_begin, int t_end, int g, const int32_t* cand, int C, int topk, int32_t* idx,
              int lim_shift, int out_stride) {
    return launch_reuse(t_begin, t_end, g, cand, C, topk, idx, nullptr, lim_shift, out_stride);
}

int emu_reuse_varlen(const int32_t* tok, const int32_t* grp, int nseq, int T, int g,
                     const int32_t* cand, int C, int topk, int32_t* idx) {
    SegTable s{};
    s.tok = tok;
    s.grp = grp;
    s.nseq = nseq;
    return launch_reuse_varlen(s, T, g, cand, C, topk, idx, nullptr);
}

int emu_decode_reuse(int B, int Gm, int maxlen, const int32_t* cache_len, const int32_t* cand,
                     int C, int topk, int32_t* idx) {
    return launch_decode_reuse(B, Gm, maxlen, cache_len, cand, C, topk, idx, nullptr);
}

int emu_window_union(const int32_t* idx, int rows, int k, int t_begin, const int32_t* positions,
                     int window, int32_t* out, int in_stride) {
    return launch_window_union(idx, rows, k, t_begin, positions, window, out, nullptr, in_stride);
}

// f32 proxies of `ngroups` groups of g members (rows of q [*, H, D], w [*, H]);
// tok / grp set: the packed groups of a ragged batch.
int emu_proxy_reduce_f32(const float* q, const float* w, int nmembers, int H, int D, int g,
                         int ngroups, float* pq, float* pw, const int32_t* tok,
                         const int32_t* grp, int nseq) {
    ReduceParams p{};
    p.dtype = PIVOT_F32;
    p.esize = 4;
    p.H = H;
    p.D = D;
    p.nmembers_total = nmembers;
    p.g = g;
    p.ngroups = ngroups;
    p.q = q;
    p.w = w;
    p.pq = pq;
    p.pw = pw;
    p.group_stride_members = g;
    if (tok) {
        p.seg.tok = tok;
        p.seg.grp = grp;
        p.seg.nseq = nseq;
    }
    return launch_proxy_reduce(p, nullptr);
}

int emu_write_ints(int32_t* dst, const int32_t* host, int n) {
    return launch_write_ints(dst, host, n, nullptr);
}

}  // extern "C"
