// profile.h -- launch bracketing for the optional kernel timing.
#pragma once

#include <cuda_runtime.h>

namespace pivot {

enum ProfKernel { PK_SCAN = 0, PK_SELECT = 1, PK_REFINE = 2, PK_REDUCE = 3, PK_REUSE = 4,
                  PK_COUNT = 5 };

bool prof_begin(int kernel, cudaStream_t s, cudaEvent_t* a, cudaEvent_t* b);
void prof_end(int kernel, cudaStream_t s, cudaEvent_t a, cudaEvent_t b, double work);
// Count a launch that is not timed (pivot_launch_count).
void count_launch();

// Run `launch` (returning cudaError_t), counted and, when timing is on,
// bracketed by events on stream `s` with `work` units attributed to it.
template <class F>
cudaError_t profiled(int kernel, double work, cudaStream_t s, F&& launch) {
    cudaEvent_t a = nullptr, b = nullptr;
    const bool on = prof_begin(kernel, s, &a, &b);
    cudaError_t e = launch();
    if (on) prof_end(kernel, s, a, b, work);
    return e;
}

}  // namespace pivot
