// runner_selftest.cpp — checks of the fiber runner itself: a warp butterfly
// sums correctly, and a CTA barrier that only some threads reach aborts.
#include <cstdlib>
#include <vector>

#include "fiber_runner.h"

extern "C" int runner_butterfly(int nthreads, float *out)
{
    FiberRunner R;
    std::vector<float> sh(nthreads);
    R.body = [&](HostX &x) {
        float v = float(x.tid() + 1);
        for (int off = 16; off > 0; off >>= 1) v += x.shfl_xor(v, off);
        sh[x.tid()] = v;
        x.sync();  // every thread sees every warp's sum after the barrier
        out[x.tid()] = sh[(x.tid() + 32) % nthreads];
    };
    R.run_block(nthreads, 0, 0);
    return 0;
}

extern "C" void runner_divergent_barrier(void)
{
    FiberRunner R;
    R.body = [&](HostX &x) {
        if (x.tid() < 16) x.sync();  // a barrier only half the block reaches
    };
    R.run_block(64, 0, 0);  // aborts
}
