// fiber_runner.h — runs a CUDA-style kernel body on the host, one fiber per
// CUDA thread, for testing kernel bodies written against an execution context.
// sync() is a block-wide barrier: every fiber runs until its next sync() (or
// its end); a barrier reached by some threads and not others aborts.
// shfl_xor() and syncwarp() are warp-level: they wait for the other 31 lanes
// of the warp only; a warp whose lanes meet different barriers aborts.
#pragma once
#include <ucontext.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <utility>
#include <functional>
#include <vector>

struct FiberRunner;

struct HostX {
    int t, bx, by;
    FiberRunner *R;
    // asynchronous 16-byte copies of this thread: committed groups, oldest
    // first, and the group being filled. A copy takes effect only when a wait
    // retires its group, so reading a buffer before waiting sees the old data.
    std::vector<std::vector<std::pair<void *, const void *>>> groups = {};
    std::vector<std::pair<void *, const void *>> open = {};
    int tid() const { return t; }
    int block() const { return bx; }
    int block_y() const { return by; }
    void sync();
    void syncwarp();
    float shfl_xor(float v, int lane_mask);
    void cp16(void *dst, const void *src) { open.push_back({dst, src}); }
    void cp_commit()
    {
        groups.push_back(open);
        open.clear();
    }
    // retire all but the newest `pending` committed groups
    void cp_wait(int pending)
    {
        while ((int)groups.size() > pending) {
            for (auto &c : groups.front()) std::memcpy(c.first, c.second, 16);
            groups.erase(groups.begin());
        }
    }
};

struct FiberRunner {
    ucontext_t sched;
    std::vector<ucontext_t> ctx;
    std::vector<std::vector<char>> stacks;
    std::vector<int> state;  // 0 runnable, 1 at a block barrier, 2 finished, 3 at a warp barrier
    std::vector<float> xchg;  // one exchange slot per thread for shuffles
    std::vector<HostX> xs;
    std::function<void(HostX &)> body;
    int cur = 0;

    static FiberRunner *&current()
    {
        static FiberRunner *r = nullptr;
        return r;
    }
    static void trampoline()
    {
        FiberRunner *R = current();
        const int t = R->cur;
        R->body(R->xs[t]);
        R->state[t] = 2;
    }
    void run_block(int nthreads, int bx, int by)
    {
        ctx.assign(nthreads, ucontext_t{});
        stacks.resize(nthreads);
        state.assign(nthreads, 0);
        xchg.assign(nthreads, 0.f);
        xs.resize(nthreads);
        current() = this;
        for (int t = 0; t < nthreads; ++t) {
            xs[t] = HostX{t, bx, by, this};
            stacks[t].resize(1 << 17);
            getcontext(&ctx[t]);
            ctx[t].uc_stack.ss_sp = stacks[t].data();
            ctx[t].uc_stack.ss_size = stacks[t].size();
            ctx[t].uc_link = &sched;
            makecontext(&ctx[t], trampoline, 0);
        }
        for (;;) {
            for (int t = 0; t < nthreads; ++t) {
                if (state[t] != 0) continue;
                cur = t;
                swapcontext(&sched, &ctx[t]);
            }
            // every fiber is now finished or waiting; release what can go on
            bool moved = false;
            for (int w0 = 0; w0 < nthreads; w0 += 32) {
                const int w1 = w0 + 32 < nthreads ? w0 + 32 : nthreads;
                int at_warp = 0, live = 0;
                for (int t = w0; t < w1; ++t) {
                    live += state[t] != 2;
                    at_warp += state[t] == 3;
                }
                if (at_warp > 0 && at_warp == live) {
                    if (live != w1 - w0) {
                        std::fprintf(stderr, "warp barrier after lanes exited in block (%d, %d)\n", bx, by);
                        std::abort();
                    }
                    for (int t = w0; t < w1; ++t) state[t] = 0;
                    moved = true;
                }
            }
            if (moved) continue;
            int done = 0, waiting = 0;
            for (int st : state) { done += st == 2; waiting += st == 1; }
            if (done == nthreads) return;
            if (waiting != nthreads) {
                std::fprintf(stderr, "barrier divergence in block (%d, %d)\n", bx, by);
                std::abort();
            }
            for (int t = 0; t < nthreads; ++t) state[t] = 0;
        }
    }
};

inline void HostX::sync()
{
    R->state[t] = 1;
    swapcontext(&R->ctx[t], &R->sched);
}

inline void HostX::syncwarp()
{
    R->state[t] = 3;
    swapcontext(&R->ctx[t], &R->sched);
}

inline float HostX::shfl_xor(float v, int lane_mask)
{
    R->xchg[t] = v;
    syncwarp();
    const float r = R->xchg[(t & ~31) | ((t & 31) ^ lane_mask)];
    syncwarp();
    return r;
}
