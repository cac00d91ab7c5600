// cbwd_host.cpp — host execution of the chunk-parallel backward's kernel bodies
// (prep, fwd_carry, bwd_carry, grad_a, grad_b) for tests; fp32 or bf16 q, k, v, dO.
#include <vector>

#include "../../gated_delta_rule_132_b200/csrc/kda_cbwd_body.cuh"
#include "fiber_runner.h"

using namespace kda::cbwd;

template <int D, typename TIn>
static void run(CbParams p, int n_chunks_alloc, float *rec_out)
{
    FiberRunner R;
    const int NS = D / WV;
    std::vector<float> smem;
    if (rec_out) {
        smem.assign(prep_smem<D>() / 4, 0.f);
        R.body = [&](HostX &x) { prep<D, TIn>(p, x, smem.data(), rec_out); };
        for (int c = 0; c < n_chunks_alloc; ++c)
            for (int h = 0; h < p.H; ++h) R.run_block(NT, c, h);
        p.rec = rec_out;
    }
    smem.assign(fwd_carry_smem<D>() / 4, 0.f);
    R.body = [&](HostX &x) { fwd_carry<D>(p, x, smem.data()); };
    for (int b = 0; b < p.N * p.H * NS; ++b) R.run_block(NT, b, 0);
    smem.assign(bwd_carry_smem<D>() / 4, 0.f);
    R.body = [&](HostX &x) { bwd_carry<D, TIn>(p, x, smem.data()); };
    for (int b = 0; b < p.N * p.H * NS; ++b) R.run_block(NT, b, 0);
    smem.assign(grad_a_smem<D>() / 4, 0.f);
    R.body = [&](HostX &x) { grad_a<D, TIn>(p, x, smem.data()); };
    for (int c = 0; c < n_chunks_alloc; ++c)
        for (int h = 0; h < p.H; ++h) R.run_block(NT, c, h);
    smem.assign(grad_b_smem<D>() / 4, 0.f);
    R.body = [&](HostX &x) { grad_b<D, TIn>(p, x, smem.data()); };
    for (int c = 0; c < n_chunks_alloc; ++c)
        for (int h = 0; h < p.H; ++h) R.run_block(NT, c, h);
}

extern "C" int cbwd_host_run(int D, int bf16, const void *q, const void *k, const void *v,
                             const void *dO, const float *log_alpha, const float *beta,
                             const float *S0, const float *dS_final, int N, int H,
                             int gate_per_channel, float scale, const int32_t *seq_start,
                             const int32_t *chunk_off, const int32_t *order, const float *rec,
                             float *Sst, float *dSst, float *Ust, float *dUst, float *scr,
                             float *gq, float *gk, float *gv, float *gla, float *gbeta,
                             float *gS0, int n_chunks_alloc, float *rec_out)
{
    CbParams p{q, k, v, dO, log_alpha, beta, S0, dS_final, N, H, gate_per_channel, scale,
               seq_start, chunk_off, order, rec, Sst, dSst, Ust, dUst, scr,
               gq, gk, gv, gla, gbeta, gS0};
    switch (D * 2 + (bf16 ? 1 : 0)) {
    case 64: run<32, float>(p, n_chunks_alloc, rec_out); return 0;
    case 65: run<32, __nv_bfloat16>(p, n_chunks_alloc, rec_out); return 0;
    case 128: run<64, float>(p, n_chunks_alloc, rec_out); return 0;
    case 129: run<64, __nv_bfloat16>(p, n_chunks_alloc, rec_out); return 0;
    case 256: run<128, float>(p, n_chunks_alloc, rec_out); return 0;
    case 257: run<128, __nv_bfloat16>(p, n_chunks_alloc, rec_out); return 0;
    default: return 1;
    }
}
