// gad_prep.cuh - the first kernel of an attention step: split of the qkv row,
// QK-norm, RoPE and the E4M3 quantise-and-scatter of k/v into the cache rows
// cache_loc[t]; the normalised queries go to the workspace (task page "Gated
// attention decode (muse_attention_decode)", section "What to compute", its
// first four lines).
#pragma once

#include "gad_kernels.cuh"

namespace gad {

// ---------------------------------------------------------------------------
// One block per (token, head group); warp w < 16 handles query head w of the
// group, warps 16 and 17 its two KV heads.  Lane l owns the RoPE pair (l,
// l + 32).  Done in double so the cache bytes match the double-precision
// definition exactly: the sum of squares runs in index order with explicit
// round-to-nearest operations (no fused multiply-add), as does the rotation.
//
// A small step's time is the latency of this kernel's loads, so every global
// value a thread needs (its two qkv elements, the position, the cache row, the
// scales and the v elements) is requested before any arithmetic: one round
// trip to memory instead of four in a row.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(PREP_THREADS) prep_kernel(const StepParams p) {
    pdl_launch_dependents();
    const int ng = p.ngrp;
    const int t = blockIdx.x / ng, c = blockIdx.x % ng;
    if (blockIdx.x == 0 && threadIdx.x == 0) *p.status = 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const __nv_bfloat16* row = p.qkv + static_cast<size_t>(t) * QKV_COLS * ng;
    const bool is_q = warp < HQ;
    const int g = warp - HQ;
    const int off = is_q ? c * OUT_COLS + warp * HD : K_OFF * ng + c * ROWB + g * HD;
    const int voff = V_OFF * ng + c * ROWB + g * HD;

    // ---- all loads first ----
    const __nv_bfloat16 bx0 = row[off + lane], bx1 = row[off + lane + 32];
    const int64_t pos = p.use_rope ? p.positions[t] : 0;
    int64_t crow = -1;
    float ksf = 1.f, vsf = 1.f;
    __nv_bfloat16 bv0 = __float2bfloat16(0.f), bv1 = bv0;
    if (!is_q) {
        crow = p.cache_loc[t];
        ksf = __ldg(p.k_scale);
        vsf = __ldg(p.v_scale);
        bv0 = row[voff + lane];
        bv1 = row[voff + lane + 32];
    }

    const double x0 = static_cast<double>(__bfloat162float(bx0));
    const double x1 = static_cast<double>(__bfloat162float(bx1));
    double ss = 0.0;
    for (int d = 0; d < 32; ++d) {
        const double v = __shfl_sync(0xffffffffu, x0, d);
        ss = __dadd_rn(ss, __dmul_rn(v, v));
    }
    for (int d = 0; d < 32; ++d) {
        const double v = __shfl_sync(0xffffffffu, x1, d);
        ss = __dadd_rn(ss, __dmul_rn(v, v));
    }
    const double r = sqrt(__dadd_rn(ss / 64.0, 1e-6));
    double u0 = x0 / r, u1 = x1 / r;
    if (is_q) {
        u0 = __dmul_rn(u0, 5.473);
        u1 = __dmul_rn(u1, 5.473);
    }
    if (p.use_rope) {
        const double phi = __dmul_rn(static_cast<double>(pos), p.inv_freq[lane]);
        double s, co;
        sincos(phi, &s, &co);
        const double r0 = __dsub_rn(__dmul_rn(u0, co), __dmul_rn(u1, s));
        const double r1 = __dadd_rn(__dmul_rn(u1, co), __dmul_rn(u0, s));
        u0 = r0;
        u1 = r1;
    }
    if (is_q) {
        __half* q = p.q_ws + (static_cast<size_t>(blockIdx.x) * HQ + warp) * HD;
        q[lane] = __double2half(u0);
        q[lane + 32] = __double2half(u1);
        return;
    }
    if (crow < 0 || crow >= p.num_rows) return;
    const double ks = static_cast<double>(ksf);
    const double vs = static_cast<double>(vsf);
    const int64_t cofs = crow * (ROWB * ng) + c * ROWB + g * HD;
    uint8_t* kd = p.k_cache + cofs;
    uint8_t* vd = p.v_cache + cofs;
    kd[lane] = __nv_cvt_float_to_fp8(__double2float_rn(u0 / ks), __NV_SATFINITE, __NV_E4M3);
    kd[lane + 32] = __nv_cvt_float_to_fp8(__double2float_rn(u1 / ks), __NV_SATFINITE, __NV_E4M3);
    const double v0 = static_cast<double>(__bfloat162float(bv0));
    const double v1 = static_cast<double>(__bfloat162float(bv1));
    vd[lane] = __nv_cvt_float_to_fp8(__double2float_rn(v0 / vs), __NV_SATFINITE, __NV_E4M3);
    vd[lane + 32] = __nv_cvt_float_to_fp8(__double2float_rn(v1 / vs), __NV_SATFINITE, __NV_E4M3);
}

}  // namespace gad
