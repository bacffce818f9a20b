// gad_combine.cuh - the last kernel of an attention step: log-sum-exp merge
// of the per-CTA partials fused with the gated output norm
//   out = rmsnorm(a) * sigmoid(gate)  -> bf16
// (task page "Gated attention decode (muse_attention_decode)", section "What
// to compute", its last line).
#pragma once

#include "gad_kernels.cuh"

namespace gad {

// ---------------------------------------------------------------------------
// Kernel 3: merge the partials of each (token, head) and apply the gated
// output norm.  One block per (token, head), over all ngrp * 16 query heads.  A request covered by many CTAs
// has many partials (a single 80K-key request spreads over ~1,200), so they
// are read in parallel: thread (sl, dq) accumulates dims 4dq..4dq+3 over
// partials sl, sl + lanes, ..., then the slot lanes are summed in shared memory.
// ---------------------------------------------------------------------------
// Block width: 1024 threads (64 slot lanes) for steps with few tokens, whose
// requests are spread over many CTAs; 256 (16 slot lanes) otherwise.
// The 1024-thread form must keep two blocks per SM (at most 32 registers a
// thread): a 16-token step launches 256 of them, one wave on 148 SMs only if
// two fit.
template <int COMB_THREADS>
__global__ void __launch_bounds__(COMB_THREADS, COMB_THREADS >= 1024 ? 2 : 1) combine_kernel(const StepParams p) {
    constexpr int COMB_SLOT_LANES = COMB_THREADS / 16;
    pdl_wait_primary();
    pdl_launch_dependents();  // a following projection may start its weight loads
    __shared__ float red_o[COMB_SLOT_LANES][HD];
    __shared__ float red_l[COMB_SLOT_LANES];
    __shared__ float red_m[COMB_THREADS / 32];
    __shared__ float red_ss[4];
    const int ng = p.ngrp, hq_all = HQ * ng;
    const int t = blockIdx.x / hq_all, hh = blockIdx.x % hq_all;  // hh = 16 * group + h
    const int h = hh % p.hp;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // list item (request, chunk, sub) and the token's place in the chunk; the
    // partial rows of an item hold p.hp query heads (sub = hh / hp)
    const int jr = t % p.L;
    const int b = ((t / p.L) * p.nchunk + jr / p.chunk) * p.nsub + hh / p.hp, j = jr % p.chunk;
    const int tp = p.meta[META_PREFIX + b];
    const int n = p.meta[META_PREFIX + b + 1] - tp;
    const int per = p.meta[META_PER];
    __nv_bfloat16* outp = p.out + static_cast<size_t>(t) * OUT_COLS * ng + hh * HD;
    if (n <= 0 || per <= 0) {  // no key in range (positions outside the contract)
        if (tid < HD) outp[tid] = __float2bfloat16(NAN);
        return;
    }
    const int c_lo = tp / per, c_hi = (tp + n - 1) / per;
    const int TL = p.tl;
    const int ns = (c_hi - c_lo + 1) * TL;
    // Partial s = (CTA c_lo + s / TL, lane s % TL); every CTA that covered some
    // of the request's tiles wrote all its lanes (a lane that saw no key of the
    // request has max -inf and is skipped).
    auto slot_base = [&](int s) {
        const int c = c_lo + s / TL, tl = s % TL;
        return ((static_cast<size_t>(c + b) * TL + tl) * p.lt + j) * p.hp + h;
    };
    // 1. global max over the slots
    float mx = -INFINITY;
    for (int s = tid; s < ns; s += COMB_THREADS) mx = fmaxf(mx, p.part_ml[slot_base(s) * 2]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red_m[warp] = mx;
    __syncthreads();
    float M = red_m[0];
#pragma unroll
    for (int w = 1; w < COMB_THREADS / 32; ++w) M = fmaxf(M, red_m[w]);
    // 2. weighted sums: thread (sl, dq) over slots sl, sl + 16, ...
    const int sl = tid / 16, dq = tid % 16;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float lsum = 0.f;
#pragma unroll 2
    for (int s = sl; s < ns; s += COMB_SLOT_LANES) {
        const size_t base = slot_base(s);
        const float ms = p.part_ml[base * 2];
        if (ms == -INFINITY) continue;
        const float w = exp2f(ms - M);
        const float4 o = *reinterpret_cast<const float4*>(p.part_o + base * HD + 4 * dq);
        acc.x += w * o.x;
        acc.y += w * o.y;
        acc.z += w * o.z;
        acc.w += w * o.w;
        lsum += w * p.part_ml[base * 2 + 1];
    }
    *reinterpret_cast<float4*>(&red_o[sl][4 * dq]) = acc;
    if (dq == 0) red_l[sl] = lsum;
    __syncthreads();
    // 3. threads 0..63: one output dim each
    if (tid < HD) {
        float o = 0.f, l = 0.f;
#pragma unroll 8
        for (int k = 0; k < COMB_SLOT_LANES; ++k) {
            o += red_o[k][tid];
            l += red_l[k];
        }
        const float a = o / l * __ldg(p.v_scale);
        float ss = a * a;
#pragma unroll
        for (int q = 16; q > 0; q >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, q);
        if (lane == 0) red_ss[warp] = ss;
        asm volatile("bar.sync 1, 64;\n" ::: "memory");
        const float tot = red_ss[0] + red_ss[1];
        const float rinv = 1.0f / sqrtf(tot * (1.0f / 64.0f) + 1e-6f);
        const float g = __bfloat162float(
            p.qkv[static_cast<size_t>(t) * QKV_COLS * ng + G_OFF * ng + hh * HD + tid]);
        outp[tid] = __float2bfloat16(a * rinv / (1.0f + expf(-g)));
    }
}

// ---------------------------------------------------------------------------
// Kernel 3b: the same merge and gated output norm with one warp per (token,
// query head), lane l holding dims 2l and 2l + 1.  For prefill blocks, whose
// items each span few CTAs, so a (token, head) has few partials and the
// block-per-(token, head) form above would spend its time on launch overhead.
// ---------------------------------------------------------------------------
constexpr int COMBW_THREADS = 256;
__global__ void __launch_bounds__(COMBW_THREADS) combine_warp_kernel(const StepParams p) {
    pdl_wait_primary();
    pdl_launch_dependents();  // a following projection may start its weight loads
    const int ng = p.ngrp, hq_all = HQ * ng;
    const int lane = threadIdx.x & 31;
    const long long gw = static_cast<long long>(blockIdx.x) * (COMBW_THREADS / 32) + (threadIdx.x >> 5);
    if (gw >= static_cast<long long>(p.B) * p.L * hq_all) return;
    const int t = static_cast<int>(gw / hq_all), hh = static_cast<int>(gw % hq_all);
    const int h = hh % p.hp;
    const int jr = t % p.L;
    const int b = ((t / p.L) * p.nchunk + jr / p.chunk) * p.nsub + hh / p.hp, j = jr % p.chunk;
    const int tp = p.meta[META_PREFIX + b];
    const int n = p.meta[META_PREFIX + b + 1] - tp;
    const int per = p.meta[META_PER];
    __nv_bfloat16* outp = p.out + static_cast<size_t>(t) * OUT_COLS * ng + hh * HD + 2 * lane;
    if (n <= 0 || per <= 0) {  // no key in range (positions outside the contract)
        outp[0] = outp[1] = __float2bfloat16(NAN);
        return;
    }
    const int c_lo = tp / per, c_hi = (tp + n - 1) / per;
    const int TL = p.tl;
    const int ns = (c_hi - c_lo + 1) * TL;
    auto slot_base = [&](int s) {
        const int c = c_lo + s / TL, tl = s % TL;
        return ((static_cast<size_t>(c + b) * TL + tl) * p.lt + j) * p.hp + h;
    };
    float M = -INFINITY;
    for (int s = lane; s < ns; s += 32) M = fmaxf(M, p.part_ml[slot_base(s) * 2]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float o0 = 0.f, o1 = 0.f, l = 0.f;
    for (int s = 0; s < ns; ++s) {
        const size_t base = slot_base(s);
        const float ms = p.part_ml[base * 2];
        if (ms == -INFINITY) continue;
        const float w = exp2f(ms - M);
        const float2 o = *reinterpret_cast<const float2*>(p.part_o + base * HD + 2 * lane);
        o0 += w * o.x;
        o1 += w * o.y;
        l += w * p.part_ml[base * 2 + 1];
    }
    const float vs = __ldg(p.v_scale);
    const float a0 = o0 / l * vs, a1 = o1 / l * vs;
    float ss = a0 * a0 + a1 * a1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rinv = 1.0f / sqrtf(ss * (1.0f / 64.0f) + 1e-6f);
    const __nv_bfloat16* gp = p.qkv + static_cast<size_t>(t) * QKV_COLS * ng + G_OFF * ng + hh * HD + 2 * lane;
    const float g0 = __bfloat162float(gp[0]), g1 = __bfloat162float(gp[1]);
    outp[0] = __float2bfloat16(a0 * rinv / (1.0f + expf(-g0)));
    outp[1] = __float2bfloat16(a1 * rinv / (1.0f + expf(-g1)));
}

}  // namespace gad
