// gad_decode2.cuh - warp-specialised split-KV decode for single-token steps over
// 64-key pages.
//
// One persistent CTA per SM: a producer warp streams 64-key tiles of the FP8
// cache into an NS-stage shared-memory ring, and 2*TL consumer warps compute
// on them.  Tile i of the CTA's share goes to tile lane i % TL; its two KV
// heads go to two consumer warps, so each consumer warp runs one head's online
// softmax over whole 64-key tiles (four 16-key MMA groups per softmax step).
//
// Loads: one 2D TMA tile (64 rows x 128 bytes, 128-byte swizzle) per K and V
// page, issued by one lane of the producer warp with completion counted on the
// stage's "full" barrier.  Consumers copy their operands to registers and
// release the stage through its "empty" barrier (one arrival per consumer warp
// of the tile) before computing.  Every wait is bounded in time; a timeout
// sets the workspace error word and the warp stops.
//
// (Random 128-byte rows of page size 1 go through decode_kernel instead: TMA
// serves small requests too slowly, and cp.async gathers from a few producer
// warps fall behind those issued by every warp of two CTAs per SM.)
//
// The MMA mapping, the shared-memory swizzle and the key permutation kappa are
// those of decode_kernel (gad_kernels.cuh).  Each consumer warp writes its own
// partial (slot (c + b) * TL + tile lane); the combine kernel merges them.
#pragma once

#include <cuda.h>

#include "gad_kernels.cuh"

namespace gad {

template <int PS, int TL, int NS>
struct Decode2Cfg {
    static_assert(PS == TILE, "one page per tile");
    static constexpr int CONSUMERS = HKV * TL;
    static constexpr int THREADS = (CONSUMERS + 1) * 32;  // + one producer warp
    static constexpr int R = 4;       // page ids are loaded R tiles ahead of their use
    static constexpr int IR = R + 2;  // ring of page ids (tiles)
    static constexpr int PITCH = ROWB;
    static constexpr int HALF = TILE * PITCH;  // K (or V) part of a stage
    static constexpr int STAGE = 2 * HALF;
    static constexpr size_t STAGES_BYTES = static_cast<size_t>(NS) * STAGE;
    static constexpr size_t BAR_BYTES = static_cast<size_t>(2 * NS) * 8;
    static constexpr size_t RING_BYTES = static_cast<size_t>(IR) * TILE * 4;
    static size_t smem_bytes(int B) {
        return 1024 /* alignment slack */ + STAGES_BYTES + BAR_BYTES + RING_BYTES +
               static_cast<size_t>(3 * B + 1) * 4;
    }
    static_assert(NS > TL + 1, "need stages beyond the ones being computed");
};

constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;  // 2 s

template <int PS, int TL, int NS>
__global__ void __launch_bounds__(Decode2Cfg<PS, TL, NS>::THREADS, 1)
    decode2_kernel(const StepParams p, const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v) {
    using C = Decode2Cfg<PS, TL, NS>;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned stages (required by the 128-byte swizzle of the TMA path)
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* stages = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES_BYTES);  // full[NS], empty[NS]
    int* ring = reinterpret_cast<int*>(smem + C::STAGES_BYTES + C::BAR_BYTES);  // [IR][64]
    int* tpre = reinterpret_cast<int*>(smem + C::STAGES_BYTES + C::BAR_BYTES + C::RING_BYTES);
    int* rlo = tpre + p.B + 1;
    int* rhi = rlo + p.B;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = p.B;

    int total, per, t0, t1;
    build_tile_list(p, tpre, rlo, rhi, C::THREADS, total, per, t0, t1);
    const int n = max(0, t1 - t0);

    const uint32_t full0 = smem_addr(bars);
    const uint32_t empty0 = smem_addr(bars + NS);
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(full0 + 8 * s, 1u);
            mbar_init(empty0 + 8 * s, 2u);
        }
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait_primary();  // q and this step's new cache rows come from the prep kernel
    if (n == 0) return;

    auto find_req = [&](int tau) {
        int lo = 0, hi = B;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (tpre[mid] <= tau) lo = mid;
            else hi = mid;
        }
        return lo;
    };
    auto advance = [&](int& tau, int& b) {
        ++tau;
        while (b < B - 1 && tau >= tpre[b + 1]) ++b;
    };

    if (warp == C::CONSUMERS) {
        // =========================== producer ===========================
        // Lane 0 loads each tile's page id R tiles ahead (into a small shared
        // ring), waits for the stage to be free and issues the two TMA loads.
        int ib = find_req(t0), it = t0;  // tile copied to shared memory
        int xb = ib, xt = t0;            // tile whose page id is loaded
        auto load_idx = [&]() {
            int v = -1;
            if (xt < t1 && lane == 0) {
                const int k0 = (rlo[xb] / TILE + (xt - tpre[xb])) * TILE;
                const int pg = k0 / PS;
                if (pg < p.max_pages) v = __ldg(p.page_table + static_cast<size_t>(xb) * p.max_pages + pg);
            }
            advance(xt, xb);
            return v;
        };
        const int64_t pages = p.num_rows / PS;
        auto page_y = [&](int pg) {
            return (pg >= 0 && pg < pages) ? pg * PS
                                           : static_cast<int>(p.num_rows < INT_MAX ? p.num_rows : INT_MAX);
        };
        int pref[C::R];
#pragma unroll
        for (int u = 0; u < C::R; ++u) pref[u] = load_idx();

        bool ok = true;
        for (int i0 = 0; i0 < n && ok; i0 += C::R) {
#pragma unroll
            for (int u = 0; u < C::R; ++u) {
                const int i = i0 + u;
                if (i >= n || !ok) break;
                if (lane == 0) ring[(i % C::IR) * TILE] = pref[u];
                pref[u] = load_idx();
                __syncwarp();
                const int s = i % NS;
                const int round = i / NS;
                if (round > 0) {
                    // every lane waits; the verdict is made warp-uniform
                    const bool got = __all_sync(
                        0xffffffffu, mbar_wait_bounded(empty0 + 8 * s, (round - 1) & 1, WAIT_LIMIT_NS));
                    if (!got) {
                        if (lane == 0) atomicExch(p.meta + META_ERROR, 1);
                        ok = false;
                        break;
                    }
                }
                if (lane == 0) {
                    const uint32_t kst = smem_addr(stages + static_cast<size_t>(s) * C::STAGE);
                    const uint32_t full = full0 + 8 * s;
                    const int y = page_y(ring[(i % C::IR) * TILE]);
                    mbar_arrive_expect_tx(full, STAGE_BYTES);
                    tma_load_2d(kst, &tmap_k, 0, y, full);
                    tma_load_2d(kst + C::HALF, &tmap_v, 0, y, full);
                }
                advance(it, ib);
            }
        }
        // Producer tail: stay until the consumers have released every stage this
        // warp filled, so no copy it issued is still in flight when it exits.
        if (ok) {
            for (int i = max(0, n - NS); i < n; ++i) {
                if (!__all_sync(0xffffffffu,
                                mbar_wait_bounded(empty0 + 8 * (i % NS), (i / NS) & 1, WAIT_LIMIT_NS))) {
                    if (lane == 0) atomicExch(p.meta + META_ERROR, 3);
                    break;
                }
            }
        }
        return;
    }

    // =========================== consumers ===========================
    const int g = warp & 1;       // KV head
    const int tl = warp >> 1;     // tile lane
    const int gid = lane >> 2, tig = lane & 3;
    const float C2 = __ldg(p.k_scale) * 0.125f * 1.4426950408889634f;
    // Row (within a 16-key group) of the MMA's logical key l, chosen per layout so
    // that the operand loads are free of bank conflicts.
    auto kap = [](int l) { return kappa(l); };
    // byte address of 16-byte chunk c of row r within a K or V half-stage
    auto caddr = [](uint32_t base, int r, int c) {
        return base + static_cast<uint32_t>(r * ROWB + ((c ^ (r & 7)) << 4));
    };
    const int krow = kap(gid);
    const int vrow0 = kap(2 * tig), vrow1 = kap(2 * tig + 1);

    float o_acc[4][4];
    float m_run[2], l_run[2];
    uint32_t qf[8];
    int cur_b = -1, lo_b = 0, hi_b = -1;

    auto begin_request = [&](int b) {
        lo_b = rlo[b];
        hi_b = rhi[b];
        const size_t t = static_cast<size_t>(b);  // single-token steps: token t = b
        const uint4* q =
            reinterpret_cast<const uint4*>(p.q_ws + (t * HQ + g * GRP + gid) * HD + 16 * tig);
        const uint4 a = q[0], c = q[1];
        qf[0] = a.x; qf[1] = a.y; qf[2] = a.z; qf[3] = a.w;
        qf[4] = c.x; qf[5] = c.y; qf[6] = c.z; qf[7] = c.w;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            m_run[e] = -INFINITY;
            l_run[e] = 0.f;
        }
#pragma unroll
        for (int dt = 0; dt < 4; ++dt)
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) o_acc[dt][c4] = 0.f;
    };

    auto flush = [&](int b) {
        const size_t slot = (static_cast<size_t>(blockIdx.x) + b) * TL + tl;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float l = l_run[e];
            l += __shfl_xor_sync(0xffffffffu, l, 4);
            l += __shfl_xor_sync(0xffffffffu, l, 8);
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            const int h = g * GRP + 2 * tig + e;
            const size_t base = (slot * p.lt + 0) * HQ + h;
            float4* dst = reinterpret_cast<float4*>(p.part_o + base * HD + 8 * gid);
            dst[0] = make_float4(o_acc[0][e], o_acc[0][2 + e], o_acc[1][e], o_acc[1][2 + e]);
            dst[1] = make_float4(o_acc[2][e], o_acc[2][2 + e], o_acc[3][e], o_acc[3][2 + e]);
            if (gid == 0) {
                p.part_ml[base * 2 + 0] = m_run[e] * C2;
                p.part_ml[base * 2 + 1] = l;
            }
        }
    };

    int ct = t0 + tl, cb = find_req(min(t0 + tl, t1 - 1));
    for (int i = tl; i < n; i += TL) {
        const int s = i % NS;
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(full0 + 8 * s, (i / NS) & 1, WAIT_LIMIT_NS))) {
            if (lane == 0) atomicExch(p.meta + META_ERROR, 2);
            cur_b = -1;
            break;
        }
        if (cb != cur_b) {
            if (cur_b >= 0) flush(cur_b);
            begin_request(cb);
            cur_b = cb;
        }
        const int k0 = (rlo[cb] / TILE + (ct - tpre[cb])) * TILE;
        const uint32_t kbase = smem_addr(stages + static_cast<size_t>(s) * C::STAGE);
        const uint32_t vbase = kbase + C::HALF;
        const bool edge = k0 < lo_b || k0 + TILE - 1 > hi_b;

        uint4 kfa[4], kfb[4];  // K rows krow, krow + 8 of each 16-key group
        uint2 vf[4][4];        // V rows vrow0, vrow1, vrow0 + 8, vrow1 + 8 of each group
        const int cpos = 4 * g + (gid >> 1);
        const uint32_t sub = static_cast<uint32_t>((gid & 1) * 8);
        auto load_k = [&](int mt) {
            const int ra = mt * 16 + krow;
            kfa[mt] = lds128(caddr(kbase, ra, 4 * g + tig));
            kfb[mt] = lds128(caddr(kbase, ra + 8, 4 * g + tig));
        };
        auto load_v = [&](int mt) {
            const int r0 = mt * 16 + vrow0, r1 = mt * 16 + vrow1;
            vf[mt][0] = lds64(caddr(vbase, r0, cpos) + sub);
            vf[mt][1] = lds64(caddr(vbase, r1, cpos) + sub);
            vf[mt][2] = lds64(caddr(vbase, r0 + 8, cpos) + sub);
            vf[mt][3] = lds64(caddr(vbase, r1 + 8, cpos) + sub);
        };
        {
            // Copy this head's operands for the whole tile into registers and
            // release the stage at once, so it is held for its load latency only.
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                load_k(mt);
                load_v(mt);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty0 + 8 * s);
            if (edge) {
                // keys outside the range get zero values (a whole page was loaded,
                // and stale codes could be NaN); their scores are masked below
#pragma unroll
                for (int mt = 0; mt < 4; ++mt) {
                    const int kb0 = k0 + mt * 16;
                    const int keys[4] = {kb0 + vrow0, kb0 + vrow1, kb0 + vrow0 + 8, kb0 + vrow1 + 8};
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        if (keys[q] < lo_b || keys[q] > hi_b) vf[mt][q] = make_uint2(0u, 0u);
                }
            }
        }

        // ---- S^T = K . Q^T over 4 groups of 16 keys ----
        float sc[4][4];
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
            const uint32_t kaw[4] = {kfa[mt].x, kfa[mt].y, kfa[mt].z, kfa[mt].w};
            const uint32_t kbw[4] = {kfb[mt].x, kfb[mt].y, kfb[mt].z, kfb[mt].w};
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) sc[mt][c4] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t a[4];
                a[0] = e4m3x2_to_f16x2(kaw[ks]);
                a[1] = e4m3x2_to_f16x2(kbw[ks]);
                a[2] = e4m3x2_to_f16x2(kaw[ks] >> 16);
                a[3] = e4m3x2_to_f16x2(kbw[ks] >> 16);
                mma_16816(sc[mt], a, qf[2 * ks], qf[2 * ks + 1]);
            }
        }
        if (edge) {
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                const int key_a = k0 + mt * 16 + krow, key_b = key_a + 8;
                if (key_a < lo_b || key_a > hi_b) sc[mt][0] = sc[mt][1] = -INFINITY;
                if (key_b < lo_b || key_b > hi_b) sc[mt][2] = sc[mt][3] = -INFINITY;
            }
        }
        // ---- online softmax (heads 2*tig + e) ----
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float mx = fmaxf(fmaxf(sc[0][e], sc[0][2 + e]), fmaxf(sc[1][e], sc[1][2 + e]));
            mx = fmaxf(mx, fmaxf(fmaxf(sc[2][e], sc[2][2 + e]), fmaxf(sc[3][e], sc[3][2 + e])));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float m_new = fmaxf(m_run[e], mx);
            const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
            const float alpha = fast_exp2((m_run[e] - m_use) * C2);
            m_run[e] = m_new;
            float lsum = l_run[e] * alpha;
#pragma unroll
            for (int dt = 0; dt < 4; ++dt) {
                o_acc[dt][e] *= alpha;
                o_acc[dt][2 + e] *= alpha;
            }
            const float mc = m_use * C2;
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                const float p0 = fast_exp2(fmaf(sc[mt][e], C2, -mc));
                const float p1 = fast_exp2(fmaf(sc[mt][2 + e], C2, -mc));
                sc[mt][e] = p0;
                sc[mt][2 + e] = p1;
                lsum += p0 + p1;
            }
            l_run[e] = lsum;
        }
        // ---- O^T += V^T . P^T ----
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
            const uint32_t pf0 = movmatrix_t(pack_f16x2(sc[mt][0], sc[mt][1]));
            const uint32_t pf1 = movmatrix_t(pack_f16x2(sc[mt][2], sc[mt][3]));
            const uint2 x0 = vf[mt][0], x1 = vf[mt][1], x2 = vf[mt][2], x3 = vf[mt][3];
#pragma unroll
            for (int dt = 0; dt < 4; ++dt) {
                const uint32_t w0 = dt < 2 ? x0.x : x0.y, w1 = dt < 2 ? x1.x : x1.y;
                const uint32_t w2 = dt < 2 ? x2.x : x2.y, w3 = dt < 2 ? x3.x : x3.y;
                const uint32_t sel = (dt & 1) ? 0x7362u : 0x5140u;
                const uint32_t p01 = __byte_perm(w0, w1, sel);
                const uint32_t p23 = __byte_perm(w2, w3, sel);
                uint32_t a[4];
                a[0] = e4m3x2_to_f16x2(p01);
                a[1] = e4m3x2_to_f16x2(p01 >> 16);
                a[2] = e4m3x2_to_f16x2(p23);
                a[3] = e4m3x2_to_f16x2(p23 >> 16);
                mma_16816(o_acc[dt], a, pf0, pf1);
            }
        }
#pragma unroll 1
        for (int k = 0; k < TL; ++k) advance(ct, cb);
    }
    if (cur_b >= 0) flush(cur_b);
}

}  // namespace gad
