#include "emu.h"
thread_local dim3 threadIdx;
dim3 blockIdx, blockDim;
static std::barrier<>* g_bar = nullptr;
static uint8_t* g_smem = nullptr;
struct Group { uint64_t vals[32]; int arrived = 0, left = 0; };
struct WarpState {
    std::mutex m;
    std::condition_variable cv;
    std::map<std::pair<unsigned, unsigned long>, Group> groups;
};
static WarpState g_warps[32];
static thread_local std::map<unsigned, unsigned long>* tl_seq = nullptr;

void __syncthreads() { g_bar->arrive_and_wait(); }
uint8_t* emu_smem() { return g_smem; }

void emu_exchange(unsigned mask, uint64_t v, uint64_t* out) {
    const unsigned lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int need = __builtin_popcount(mask);
    WarpState& ws = g_warps[w];
    const unsigned long seq = (*tl_seq)[mask]++;
    std::unique_lock<std::mutex> lk(ws.m);
    Group& G = ws.groups[{mask, seq}];
    G.vals[lane] = v;
    if (++G.arrived == need) ws.cv.notify_all();
    else if (!ws.cv.wait_for(lk, std::chrono::seconds(20), [&] { return G.arrived == need; }))
        EMU_FAIL("warp %u collective (mask %08x seq %lu) never completed: %d of %d lanes", w, mask, seq,
                 G.arrived, need);
    memcpy(out, G.vals, sizeof(G.vals));
    if (++G.left == need) ws.groups.erase({mask, seq});
}

void emu_launch(int nblocks, int nthreads, size_t smem_bytes, const std::function<void()>& fn) {
    blockDim.x = nthreads;
    for (int b = 0; b < nblocks; ++b) {
        blockIdx.x = b;
        g_smem = (uint8_t*)malloc(smem_bytes);
        { const char* pv = getenv("EMU_POISON"); int pat = pv ? atoi(pv) : 0xA5; if (pat < 0) { for (size_t i = 0; i < smem_bytes; ++i) g_smem[i] = (uint8_t)rand(); } else memset(g_smem, pat, smem_bytes); }
        std::barrier<> bar(nthreads);
        g_bar = &bar;
        std::vector<std::thread> th;
        th.reserve(nthreads);
        for (int t = 0; t < nthreads; ++t)
            th.emplace_back([&, t] {
                threadIdx.x = t;
                std::map<unsigned, unsigned long> seq;
                tl_seq = &seq;
                fn();
                // a returning thread leaves the block barrier
                g_bar->arrive_and_drop();
            });
        for (auto& x : th) x.join();
        free(g_smem);
        g_smem = nullptr;
    }
}
