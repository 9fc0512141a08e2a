// Host emulation of the CUDA features the select kernel uses: one block at a
// time, one std::thread per CUDA thread, barriers for __syncthreads and
// mask-keyed exchanges for the warp collectives.  For finding faults on CPU
// (ASan/UBSan) -- not a product path.
#pragma once
#include <cstdint>
#include <cstring>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <barrier>
#include <condition_variable>
#include <functional>
#include <map>
#include <mutex>
#include <thread>
#include <vector>

#define __device__
#define __host__
#define __global__
#define __forceinline__ inline
#define __noinline__ __attribute__((noinline))
#define __launch_bounds__(...)
#define __align__(n) alignas(n)
#define __shared__ static
#define __restrict__

typedef int cudaError_t;
typedef void* cudaStream_t;
constexpr int cudaSuccess = 0;
constexpr int cudaErrorInvalidValue = 1;
constexpr int cudaFuncAttributeMaxDynamicSharedMemorySize = 8;
constexpr int cudaFuncAttributePreferredSharedMemoryCarveout = 9;
constexpr int cudaSharedmemCarveoutMaxShared = 100;
struct CUtensorMap { char b[128]; };
template <class F> inline cudaError_t cudaFuncSetAttribute(F, int, int) { return cudaSuccess; }
inline cudaError_t cudaGetLastError() { return cudaSuccess; }

struct dim3 { unsigned x = 0, y = 0, z = 0; };
extern thread_local dim3 threadIdx;
extern dim3 blockIdx, blockDim;

struct alignas(16) float4 { float x, y, z, w; };
inline float4 make_float4(float a, float b, float c, float d) { return {a, b, c, d}; }

#define EMU_FAIL(...) do { fprintf(stderr, "EMU FAULT: " __VA_ARGS__); fprintf(stderr, "\n"); abort(); } while (0)

inline float4 __ldcs(const float4* p) {
    if ((uintptr_t)p & 15) EMU_FAIL("misaligned float4 load %p", (const void*)p);
    return *p;
}

inline uint32_t __float_as_uint(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
inline float __uint_as_float(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
inline int __popc(unsigned x) { return __builtin_popcount(x); }
inline int __ffs(unsigned x) { return __builtin_ffs((int)x); }
template <class A, class B> inline auto min(A a, B b) -> decltype(a + b) { return a < b ? a : b; }
template <class A, class B> inline auto max(A a, B b) -> decltype(a + b) { return a < b ? b : a; }

template <class T> inline void emu_check_align(T* p) {
    if ((uintptr_t)p % sizeof(T)) EMU_FAIL("misaligned %zu-byte atomic %p", sizeof(T), (void*)p);
}
template <class T> inline T atomicAdd(T* p, T v) { emu_check_align(p); return __atomic_fetch_add(p, v, __ATOMIC_SEQ_CST); }
inline unsigned atomicAdd(unsigned* p, int v) { return atomicAdd(p, (unsigned)v); }
template <class T> inline T atomicOr(T* p, T v) { emu_check_align(p); return __atomic_fetch_or(p, v, __ATOMIC_SEQ_CST); }
template <class T> inline T atomicMin(T* p, T v) {
    emu_check_align(p);
    T o = __atomic_load_n(p, __ATOMIC_SEQ_CST);
    while (v < o && !__atomic_compare_exchange_n(p, &o, v, false, __ATOMIC_SEQ_CST, __ATOMIC_SEQ_CST)) {}
    return o;
}
template <class T> inline T atomicMax(T* p, T v) {
    emu_check_align(p);
    T o = __atomic_load_n(p, __ATOMIC_SEQ_CST);
    while (v > o && !__atomic_compare_exchange_n(p, &o, v, false, __ATOMIC_SEQ_CST, __ATOMIC_SEQ_CST)) {}
    return o;
}

void __syncthreads();
void emu_exchange(unsigned mask, uint64_t v, uint64_t* out);

template <class T> inline uint64_t emu_pack(T v) { uint64_t r = 0; memcpy(&r, &v, sizeof(T)); return r; }
template <class T> inline T emu_unpack(uint64_t r) { T v; memcpy(&v, &r, sizeof(T)); return v; }

inline unsigned emu_lane() { return threadIdx.x & 31; }
inline void __syncwarp(unsigned mask = 0xffffffffu) { uint64_t v[32]; emu_exchange(mask, 0, v); }
inline int __clz(unsigned x) { return x ? __builtin_clz(x) : 32; }
inline int __clzll(long long x) { return x ? __builtin_clzll((unsigned long long)x) : 64; }
inline void emu_check_mask(unsigned mask) {
    if (!((mask >> emu_lane()) & 1)) EMU_FAIL("lane %u not in its own mask %08x", emu_lane(), mask);
}
inline unsigned __ballot_sync(unsigned mask, bool p) {
    emu_check_mask(mask);
    uint64_t v[32];
    emu_exchange(mask, p ? 1 : 0, v);
    unsigned r = 0;
    for (int l = 0; l < 32; ++l) if (((mask >> l) & 1) && v[l]) r |= 1u << l;
    return r;
}
inline bool __any_sync(unsigned mask, bool p) { return __ballot_sync(mask, p) != 0; }
inline bool __all_sync(unsigned mask, bool p) { return __ballot_sync(mask, p) == mask; }
template <class T> inline T __shfl_sync(unsigned mask, T x, int src) {
    emu_check_mask(mask);
    uint64_t v[32];
    emu_exchange(mask, emu_pack(x), v);
    src &= 31;
    if (!((mask >> src) & 1)) EMU_FAIL("shfl from lane %d outside mask %08x", src, mask);
    return emu_unpack<T>(v[src]);
}
template <class T> inline T __shfl_xor_sync(unsigned mask, T x, int o) {
    emu_check_mask(mask);
    uint64_t v[32];
    emu_exchange(mask, emu_pack(x), v);
    const int s = (int)(emu_lane() ^ (unsigned)o) & 31;
    if (!((mask >> s) & 1)) EMU_FAIL("shfl_xor from lane %d outside mask", s);
    return emu_unpack<T>(v[s]);
}
template <class T> inline T __shfl_up_sync(unsigned mask, T x, int o) {
    emu_check_mask(mask);
    uint64_t v[32];
    emu_exchange(mask, emu_pack(x), v);
    const int l = (int)emu_lane();
    if (l < o) return x;
    if (!((mask >> (l - o)) & 1)) EMU_FAIL("shfl_up from lane outside mask");
    return emu_unpack<T>(v[l - o]);
}
template <class T> inline unsigned __match_any_sync(unsigned mask, T x) {
    emu_check_mask(mask);
    uint64_t v[32];
    emu_exchange(mask, emu_pack(x), v);
    const uint64_t me = emu_pack(x);
    unsigned r = 0;
    for (int l = 0; l < 32; ++l) if (((mask >> l) & 1) && v[l] == me) r |= 1u << l;
    return r;
}

// run fn for nblocks blocks of nthreads threads with `smem_bytes` of dynamic
// shared memory (heap-allocated at exactly that size, filled with 0xA5)
void emu_launch(int nblocks, int nthreads, size_t smem_bytes, const std::function<void()>& fn);
uint8_t* emu_smem();
