// gad_oproj.cuh - the output projection that follows the attention step in
// the decoder layer: a = out @ o^T (the pages "Decode layer
// (muse_decode_layer)" and "Prefill layer (muse_prefill_layer)", section
// "What to compute": a = (rmsnorm(attention(q)) * sigmoid(g)) @ o.T, the
// all-reduce after it being the identity on one GPU).
//
//   out  bf16 [T, K]   the step's gated, normalised attention output
//   o    bf16 [N, K]   the projection weight, row n = hidden unit n
//   a    bf16 [T, N]   fp32 accumulation, one rounding
//
// One CTA per (128 hidden rows, up to 256 tokens): D[n][t] = sum_k o[n][k]
// out[t][k] is one tcgen05 MMA chain (M 128 = hidden rows, N = tokens, K in
// 64-wide steps) with both operands staged by 2D TMA tile loads (128-byte
// swizzle) through a ring of as many stages as the shared memory holds for
// the token tile (10 at 32 tokens), the accumulator in tensor memory.  Warp 0
// lane 0 issues the loads, warp 1 the MMAs, and all four warps read the
// accumulator back (lane = hidden row) and store a column of a per token.
//
// The kernel follows the combine kernel under programmatic dependent launch:
// its first weight stages are requested before it waits for the attention
// kernels, so the weight stream (the bulk of its bytes) overlaps them.
#pragma once

#include <cuda.h>

#include "gad_kernels.cuh"
#include "gad_tc.cuh"

namespace gad {
namespace opj {

constexpr int BM = 128;                   // hidden rows per CTA (MMA M)
constexpr int BK = 64;                    // contraction per stage: one 128-byte row of bf16
constexpr int TT_MAX = 256;               // tokens per CTA (MMA N)
constexpr int NSTG_MAX = 16;              // ring stages at most
constexpr int SMEM_BUDGET = 200 * 1024;   // bytes of ring per CTA
constexpr int THREADS = 128;
constexpr int W_STAGE = BM * BK * 2;      // 16 KB of weight rows per stage

__host__ __device__ constexpr int x_stage(int tt) { return tt * BK * 2; }  // token rows per stage
__host__ __device__ constexpr int ctrl_bytes() { return 8 * (2 * NSTG_MAX + 1) + 8; }  // barriers, TMEM, flag
__host__ __device__ constexpr int stages(int tt, int nk) {  // ring stages for a token tile
    const int fit = SMEM_BUDGET / (W_STAGE + x_stage(tt));
    const int s = fit < NSTG_MAX ? fit : NSTG_MAX;
    return s < nk ? s : nk;
}
__host__ __device__ constexpr size_t smem_bytes(int tt, int nstg) {
    return 1024 + static_cast<size_t>(nstg) * (W_STAGE + x_stage(tt)) + ctrl_bytes();
}
__host__ __device__ constexpr uint32_t tmem_cols(int tt) {  // a power of two >= 32
    return tt <= 32 ? 32u : tt <= 64 ? 64u : tt <= 128 ? 128u : 256u;
}


}  // namespace opj

struct OprojParams {
    __nv_bfloat16* a;  // [T, N]
    int T, K, N;
    int tt;            // tokens per CTA: a multiple of 16, at most 256
    int nstg;          // ring stages (stages(tt, K / BK))
    int* err;          // status word: STATUS_OPROJ_WAIT is or-ed in if a bounded wait gave up
};

__global__ void __launch_bounds__(opj::THREADS, 1)
    oproj_kernel(const __grid_constant__ CUtensorMap w_map, const __grid_constant__ CUtensorMap x_map,
                 const OprojParams p) {
    using namespace opj;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    const int xs = x_stage(p.tt);
    const int NSTG = p.nstg;
    const uint32_t wbuf = smem_addr(smem);                         // [NSTG][128 rows][128 B]
    const uint32_t xbuf = wbuf + NSTG * W_STAGE;                   // [NSTG][tt rows][128 B]
    uint8_t* ctrl = smem + NSTG * (W_STAGE + xs);
    const uint32_t bar0 = smem_addr(ctrl);
    auto FULL = [&](int s) { return bar0 + 8u * static_cast<uint32_t>(s); };
    auto EMPTY = [&](int s) { return bar0 + 8u * static_cast<uint32_t>(NSTG + s); };
    const uint32_t DONE = bar0 + 8u * (2 * NSTG);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 8 * (2 * NSTG + 1));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl + 8 * (2 * NSTG + 1) + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n0 = blockIdx.x * BM, t0 = blockIdx.y * p.tt;
    const int nk = p.K / BK;
    const uint32_t ncols = tmem_cols(p.tt);

    if (tid == 0) {
        for (int s = 0; s < NSTG; ++s) {
            mbar_init(FULL(s), 1);  // the producer's arrive with the stage's expected bytes
            mbar_init(EMPTY(s), 1);
        }
        mbar_init(DONE, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 1) {
        tc_alloc(smem_addr(tmem_slot), ncols);
        tc_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---- loads: weights of the first stages before the attention step has
            // finished (they do not depend on it), then its output ----
            const uint32_t bytes = static_cast<uint32_t>(W_STAGE + xs);
            const int first = nk < NSTG ? nk : NSTG;
            for (int kc = 0; kc < first; ++kc) {
                mbar_arrive_expect_tx(FULL(kc), bytes);
                tma_load_2d(wbuf + kc * W_STAGE, &w_map, kc * BK, n0, FULL(kc));
            }
            pdl_wait_primary();
            for (int kc = 0; kc < first; ++kc) tma_load_2d(xbuf + kc * xs, &x_map, kc * BK, t0, FULL(kc));
            int issued = first;  // stages [0, issued) have their loads in flight or landed
            for (int kc = NSTG; kc < nk; ++kc) {
                const int s = kc % NSTG;
                if (!wait_bounded(EMPTY(s), (kc / NSTG - 1) & 1, abort_flag)) break;
                mbar_arrive_expect_tx(FULL(s), bytes);
                tma_load_2d(wbuf + s * W_STAGE, &w_map, kc * BK, n0, FULL(s));
                tma_load_2d(xbuf + s * xs, &x_map, kc * BK, t0, FULL(s));
                issued = kc + 1;
            }
            // Every load issued must land before the CTA leaves (its shared
            // memory is the destination): wait for the last one of each stage,
            // also after an abort.  Without an abort they have all been
            // consumed by now and these waits return at once.
            for (int kc = issued > NSTG ? issued - NSTG : 0; kc < issued; ++kc)
                wait_bounded(FULL(kc % NSTG), (kc / NSTG) & 1, abort_flag, false, TEARDOWN_LIMIT_NS);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---- MMAs: whole warp, warp-uniform control flow, one elected lane ----
        const uint32_t idesc = idesc_bf16_f32(BM, p.tt, 0);  // B (tokens x K) K-major
        for (int kc = 0; kc < nk; ++kc) {
            const int s = kc % NSTG;
            const bool got = wait_bounded(FULL(s), (kc / NSTG) & 1, abort_flag);
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            const uint32_t wa = wbuf + s * W_STAGE, xa = xbuf + s * xs;
            const uint64_t ad[4] = {smem_desc_sw128(wa), smem_desc_sw128(wa + 32), smem_desc_sw128(wa + 64),
                                    smem_desc_sw128(wa + 96)};
            const uint64_t bd[4] = {smem_desc_sw128(xa), smem_desc_sw128(xa + 32), smem_desc_sw128(xa + 64),
                                    smem_desc_sw128(xa + 96)};
            tc_mma_ss4(tmem, ad, bd, idesc, kc > 0 ? 1u : 0u);
            tc_commit(EMPTY(s));
        }
        tc_commit(DONE);  // every MMA issued above (or none) is done before it fires
    }

    // ---- epilogue: lane = hidden row, columns = tokens ----
    // (every MMA issued, also before an abort, is done before tensor memory is
    // read or freed)
    const bool done = wait_bounded(DONE, 0, abort_flag, false, TEARDOWN_LIMIT_NS);
    tc_fence_after();
    if (__all_sync(0xffffffffu, done && !*abort_flag)) {  // warp-uniform: tcgen05.ld is collective
        const int n = n0 + warp * 32 + lane;
        const uint32_t row = tmem + (static_cast<uint32_t>(32 * warp) << 16);
        uint32_t v[32];
        for (int c0 = 0; c0 < p.tt; c0 += 32) {
            tc_ld32(row + static_cast<uint32_t>(c0), v);
            tc_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int t = t0 + c0 + j;
                if (c0 + j < p.tt && t < p.T)
                    p.a[static_cast<size_t>(t) * p.N + n] = __float2bfloat16(__uint_as_float(v[j]));
            }
        }
    }

    // ---- teardown ----
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tc_dealloc(tmem, ncols);
    }
    if (tid == 0 && *abort_flag) {
        pdl_wait_primary();  // the step's first kernel has cleared the status word
        atomicOr(p.err, STATUS_OPROJ_WAIT);
    }
    pdl_launch_dependents();
}

}  // namespace gad
