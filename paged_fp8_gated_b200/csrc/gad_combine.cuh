// gad_combine.cuh - the last kernel of an attention step: log-sum-exp merge
// of the per-CTA partials fused with the gated output norm
//   out = rmsnorm(a) * sigmoid(gate)  -> bf16
// (task page "Gated attention decode (muse_attention_decode)", section "What
// to compute", its last line).
#pragma once

#include "gad_kernels.cuh"

namespace gad {

// Three forms of the same merge, chosen by the launcher:
//   combine_kernel<1024, MINB>  steps of at most 16 (token, group) pairs
//   combine_kernel<256, 8>      other single-token steps
//   combine_warp4_kernel        other verify blocks
//   combine_warp_kernel         prefill blocks
// Each merges in one pass: a lane keeps a running max over the partials it
// reads (rescaling its sums when the max rises), and the lanes' sums are
// rescaled to their common max only when they are added together.
//
// ---------------------------------------------------------------------------
// Kernel 3: merge the partials of each (token, head) and apply the gated
// output norm.  One block per (token, head), over all ngrp * 16 query heads.
// A request covered by many CTAs has many partials (a single 80K-key request
// spreads over ~1,200), so they are read in parallel: thread (sl, dq)
// accumulates dims 4dq..4dq+3 over partials sl, sl + lanes, ..., then the
// slot lanes are summed in shared memory.
// ---------------------------------------------------------------------------
// Block width: 1024 threads (64 slot lanes) for steps with few tokens, whose
// requests are spread over many CTAs; 256 (16 slot lanes) otherwise.
// MINB blocks per SM: a grid of at most one block per SM (a 1-token step: 16
// blocks) runs each block faster with registers to spare (47 a thread); a
// 16-token step launches 256 blocks of 1024 threads, one wave on 148 SMs only
// if two fit (at most 32 registers a thread), and so do 8 blocks of 256.
template <int COMB_THREADS, int MINB>
__global__ void __launch_bounds__(COMB_THREADS, MINB) combine_kernel(const StepParams p) {
    constexpr int COMB_SLOT_LANES = COMB_THREADS / 16;
    __shared__ float red_o[COMB_SLOT_LANES][HD];
    __shared__ float red_l[COMB_SLOT_LANES];
    __shared__ float red_m[COMB_THREADS / 32];
    __shared__ float red_ss[4];
    __shared__ float gate_s[HD + 1];  // the gate row and v_scale (step inputs)
    const int ng = p.ngrp, hq_all = HQ * ng;
    const int t = blockIdx.x / hq_all, hh = blockIdx.x % hq_all;  // hh = 16 * group + h
    const int h = hh % p.hp;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // The gate and v_scale are inputs, not results of the earlier kernels: fetch
    // them while those finish (parked in shared memory, off the register budget).
    if (tid < HD)
        gate_s[tid] = __bfloat162float(p.qkv[static_cast<size_t>(t) * QKV_COLS * ng + G_OFF * ng + hh * HD + tid]);
    else if (tid == HD)
        gate_s[HD] = __ldg(p.v_scale);
    pdl_wait_primary();
    pdl_launch_dependents();  // a following projection may start its weight loads
    // list item (request, chunk, sub) and the token's place in the chunk; the
    // partial rows of an item hold p.hp query heads (sub = hh / hp)
    const int jr = t % p.L;
    const int b = ((t / p.L) * p.nchunk + jr / p.chunk) * p.nsub + hh / p.hp, j = jr % p.chunk;
    const int tp = p.meta[META_PREFIX + b];
    const int n = p.meta[META_PREFIX + b + 1] - tp;
    const int per = p.meta[META_PER];
    // the output row is addressed only at the end (a 64-bit pointer held across
    // the loops would not fit a 32-register budget)
    auto outp = [&]() { return p.out + static_cast<size_t>(t) * OUT_COLS * ng + hh * HD; };
    if (n <= 0 || per <= 0) {  // no key in range (positions outside the contract)
        if (tid < HD) outp()[tid] = __float2bfloat16(NAN);
        return;
    }
    const int c_lo = tp / per, c_hi = (tp + n - 1) / per;
    const int TL = p.tl;
    const int ns = (c_hi - c_lo + 1) * TL;
    // Partial s = (CTA c_lo + s / TL, lane s % TL) sits in slot (c + b) * TL + lane
    // = (c_lo + b) * TL + s; every CTA that covered some of the request's tiles
    // wrote all its lanes (a lane that saw no key of the request has max -inf and
    // is skipped).  Row (token j, head h) of a slot: slot * lt * hp + j * hp + h.
    // 32-bit row indices: the workspace holds fewer than 2^25 partial rows
    const int slot0 = (c_lo + b) * TL;
    const int stride = p.lt * p.hp, row0 = j * p.hp + h;
    auto slot_base = [&](int s) { return (slot0 + s) * stride + row0; };
    // 1. weighted sums in one pass: thread (sl, dq) over slots sl, sl + lanes,
    // ..., each slot lane keeping its own running max (weights <= 1), so no
    // separate pass over the maxima precedes the sums
    const int sl = tid / 16, dq = tid % 16;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float lsum = 0.f, mrun = -INFINITY;
    // partials in flight per thread: 4 with the registers of one block per SM
    // (the loop is bound by L2 latency when 16 blocks merge ~1,200 partials each)
#pragma unroll(MINB == 1 ? 4 : 2)
    for (int s = sl; s < ns; s += COMB_SLOT_LANES) {
        const int base = slot_base(s);
        // All three loads are issued before the test (every slot below ns was
        // written by this step), so unrolled iterations overlap their latency.
        const float2 ml = *reinterpret_cast<const float2*>(p.part_ml + base * 2);
        const float4 o = *reinterpret_cast<const float4*>(p.part_o + base * HD + 4 * dq);
        if (ml.x != -INFINITY) {
            if (ml.x > mrun) {  // rescale what this lane has summed so far
                const float a = exp2f(mrun - ml.x);  // 0 while nothing was summed
                acc.x *= a;
                acc.y *= a;
                acc.z *= a;
                acc.w *= a;
                lsum *= a;
                mrun = ml.x;
            }
            const float w = exp2f(ml.x - mrun);
            acc.x += w * o.x;
            acc.y += w * o.y;
            acc.z += w * o.z;
            acc.w += w * o.w;
            lsum += w * ml.y;
        }
    }
    // 2. block max of the lanes' maxima (a warp holds two slot lanes), then
    // each lane's sums rescaled to it
    float mx = fmaxf(mrun, __shfl_xor_sync(0xffffffffu, mrun, 16));
    if (lane == 0) red_m[warp] = mx;
    __syncthreads();
    float M = red_m[0];
#pragma unroll
    for (int w = 1; w < COMB_THREADS / 32; ++w) M = fmaxf(M, red_m[w]);
    const float sc = mrun == -INFINITY ? 0.f : exp2f(mrun - M);
    acc.x *= sc;
    acc.y *= sc;
    acc.z *= sc;
    acc.w *= sc;
    *reinterpret_cast<float4*>(&red_o[sl][4 * dq]) = acc;
    if (dq == 0) red_l[sl] = lsum * sc;
    __syncthreads();
    // 3. threads 0..63: one output dim each
    if (tid < HD) {
        float o = 0.f, l = 0.f;
#pragma unroll 8
        for (int k = 0; k < COMB_SLOT_LANES; ++k) {
            o += red_o[k][tid];
            l += red_l[k];
        }
        const float a = o / l * gate_s[HD];
        float ss = a * a;
#pragma unroll
        for (int q = 16; q > 0; q >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, q);
        if (lane == 0) red_ss[warp] = ss;
        asm volatile("bar.sync 1, 64;\n" ::: "memory");
        const float tot = red_ss[0] + red_ss[1];
        const float rinv = 1.0f / sqrtf(tot * (1.0f / 64.0f) + 1e-6f);
        const float g = gate_s[tid];
        outp()[tid] = __float2bfloat16(a * rinv / (1.0f + expf(-g)));
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
    const int ng = p.ngrp, hq_all = HQ * ng;
    const int lane = threadIdx.x & 31;
    const long long gw = static_cast<long long>(blockIdx.x) * (COMBW_THREADS / 32) + (threadIdx.x >> 5);
    const bool live = gw < static_cast<long long>(p.B) * p.L * hq_all;
    const int t = live ? static_cast<int>(gw / hq_all) : 0, hh = live ? static_cast<int>(gw % hq_all) : 0;
    // the gate and v_scale are step inputs: fetched while the earlier kernels finish
    __nv_bfloat162 gv = __floats2bfloat162_rn(0.f, 0.f);
    float vs = 0.f;
    if (live) {
        gv = *reinterpret_cast<const __nv_bfloat162*>(p.qkv + static_cast<size_t>(t) * QKV_COLS * ng +
                                                       G_OFF * ng + hh * HD + 2 * lane);
        vs = __ldg(p.v_scale);
    }
    pdl_wait_primary();
    pdl_launch_dependents();  // a following projection may start its weight loads
    if (!live) return;
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
    const int slot0 = (c_lo + b) * TL;  // slot of partial s: slot0 + s (32-bit row indices)
    const int stride = p.lt * p.hp, row0 = j * p.hp + h;
    auto slot_base = [&](int s) { return (slot0 + s) * stride + row0; };
    // one pass with a running max (the same for every lane: all lanes walk the
    // same partials); loads first, test after
    float o0 = 0.f, o1 = 0.f, l = 0.f, mrun = -INFINITY;
#pragma unroll 2
    for (int s = 0; s < ns; ++s) {
        const int base = slot_base(s);
        const float2 ml = *reinterpret_cast<const float2*>(p.part_ml + base * 2);
        const float2 o = *reinterpret_cast<const float2*>(p.part_o + base * HD + 2 * lane);
        if (ml.x != -INFINITY) {
            if (ml.x > mrun) {
                const float a = exp2f(mrun - ml.x);  // 0 while nothing was summed
                o0 *= a;
                o1 *= a;
                l *= a;
                mrun = ml.x;
            }
            const float w = exp2f(ml.x - mrun);
            o0 += w * o.x;
            o1 += w * o.y;
            l += w * ml.y;
        }
    }
    const float a0 = o0 / l * vs, a1 = o1 / l * vs;
    float ss = a0 * a0 + a1 * a1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rinv = 1.0f / sqrtf(ss * (1.0f / 64.0f) + 1e-6f);
    const float g0 = __low2float(gv), g1 = __high2float(gv);
    outp[0] = __float2bfloat16(a0 * rinv / (1.0f + expf(-g0)));
    outp[1] = __float2bfloat16(a1 * rinv / (1.0f + expf(-g1)));
}

// ---------------------------------------------------------------------------
// Kernel 3c: one warp per (token, query head) in four slot groups of eight
// lanes, lane (g, dl) holding dims 8dl..8dl+7 of slots g, g + 4, ...; the
// groups are summed with shuffles.  For verify blocks: thousands of (token,
// head) pairs with tens of partials each, where the block form above leaves
// most of its threads idle behind barriers and the single-slot warp form
// walks the partials one by one.
// ---------------------------------------------------------------------------
constexpr int COMBW4_THREADS = 256;
__global__ void __launch_bounds__(COMBW4_THREADS) combine_warp4_kernel(const StepParams p) {
    const int ng = p.ngrp, hq_all = HQ * ng;
    const int lane = threadIdx.x & 31, g = lane >> 3, dl = lane & 7;
    const long long gw = static_cast<long long>(blockIdx.x) * (COMBW4_THREADS / 32) + (threadIdx.x >> 5);
    const bool live = gw < static_cast<long long>(p.B) * p.L * hq_all;
    const int t = live ? static_cast<int>(gw / hq_all) : 0, hh = live ? static_cast<int>(gw % hq_all) : 0;
    const int d0 = 8 * dl + 2 * g;  // the two output dims this lane writes
    // the gate and v_scale are step inputs: fetched while the earlier kernels finish
    __nv_bfloat162 gv = __floats2bfloat162_rn(0.f, 0.f);
    float vs = 0.f;
    if (live) {
        gv = *reinterpret_cast<const __nv_bfloat162*>(p.qkv + static_cast<size_t>(t) * QKV_COLS * ng +
                                                       G_OFF * ng + hh * HD + d0);
        vs = __ldg(p.v_scale);
    }
    pdl_wait_primary();
    pdl_launch_dependents();  // a following projection may start its weight loads
    if (!live) return;
    const int h = hh % p.hp;
    const int jr = t % p.L;
    const int b = ((t / p.L) * p.nchunk + jr / p.chunk) * p.nsub + hh / p.hp, j = jr % p.chunk;
    const int tp = p.meta[META_PREFIX + b];
    const int n = p.meta[META_PREFIX + b + 1] - tp;
    const int per = p.meta[META_PER];
    __nv_bfloat162* outp = reinterpret_cast<__nv_bfloat162*>(p.out + static_cast<size_t>(t) * OUT_COLS * ng +
                                                             hh * HD + d0);
    if (n <= 0 || per <= 0) {  // no key in range (positions outside the contract)
        *outp = __floats2bfloat162_rn(NAN, NAN);
        return;
    }
    const int c_lo = tp / per, c_hi = (tp + n - 1) / per;
    const int TL = p.tl;
    const int ns = (c_hi - c_lo + 1) * TL;
    const int slot0 = (c_lo + b) * TL;  // slot of partial s: slot0 + s (32-bit row indices)
    const int stride = p.lt * p.hp, row0 = j * p.hp + h;
    auto slot_base = [&](int s) { return (slot0 + s) * stride + row0; };
    // one pass: each slot group keeps its own running max, rescaled to the
    // warp's max before the groups are summed
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float l = 0.f, mrun = -INFINITY;
#pragma unroll 2
    for (int s = g; s < ns; s += 4) {
        const int base = slot_base(s);
        // loads first (every slot below ns was written by this step), test after
        const float2 ml = *reinterpret_cast<const float2*>(p.part_ml + base * 2);
        const float4* src = reinterpret_cast<const float4*>(p.part_o + base * HD + 8 * dl);
        const float4 x = src[0], y = src[1];
        if (ml.x != -INFINITY) {
            if (ml.x > mrun) {  // rescale what this group has summed so far
                const float a = exp2f(mrun - ml.x);  // 0 while nothing was summed
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] *= a;
                l *= a;
                mrun = ml.x;
            }
            const float w = exp2f(ml.x - mrun);
            acc[0] += w * x.x;
            acc[1] += w * x.y;
            acc[2] += w * x.z;
            acc[3] += w * x.w;
            acc[4] += w * y.x;
            acc[5] += w * y.y;
            acc[6] += w * y.z;
            acc[7] += w * y.w;
            l += w * ml.y;
        }
    }
    // the warp's max over the four groups (lanes of a group agree), then rescale
    float M = fmaxf(mrun, __shfl_xor_sync(0xffffffffu, mrun, 8));
    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 16));
    const float sc = mrun == -INFINITY ? 0.f : exp2f(mrun - M);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] *= sc;
    l *= sc;
#pragma unroll
    for (int o = 8; o <= 16; o <<= 1) {  // sum the four slot groups
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
        l += __shfl_xor_sync(0xffffffffu, l, o);
    }
    float ss = 0.f, a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float a = acc[i] / l * vs;
        ss += a * a;
        if (i == 2 * g) a0 = a;  // unrolled selects: no local-memory indexing
        if (i == 2 * g + 1) a1 = a;
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);  // over the 8 dim lanes
    const float rinv = 1.0f / sqrtf(ss * (1.0f / 64.0f) + 1e-6f);
    const float g0 = __low2float(gv), g1 = __high2float(gv);
    *outp = __floats2bfloat162_rn(a0 * rinv / (1.0f + expf(-g0)), a1 * rinv / (1.0f + expf(-g1)));
}

}  // namespace gad
