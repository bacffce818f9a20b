// gad_verify_tc.cuh - verify-block decode (q_len 2..8) on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory).
//
// Method: task page "Gated attention decode (muse_attention_decode)", section
// "What to compute" (S = q.K^T / 8 over the request's keys up to the token's
// position, softmax, P.V); the verify-block shapes from its section "Shapes".
//
// One tile = 64 keys of one request, aligned to absolute key index (the same
// tile list and partial slots as decode_kernel: CTA c takes tiles
// [c*per, (c+1)*per) and writes one (o, max, sum) partial per request it
// touches into slot c + b).
//
// Rows.  The 8 tokens x 16 query heads of a request are the 128 rows of the
// MMA (row r: KV head g = r / 64, token j = (r / 8) % 8, query head 8g + r % 8).
// Both KV heads share one MMA by padding the contraction: the A operand of
// S = A . B^T is [q | 0] for KV head 0 and [0 | q] for KV head 1 (K = 128),
// and B is the whole converted cache row [k_head0 | k_head1].  For P.V the
// output is 128 rows x (64 dims of head 0 | 64 dims of head 1); row r keeps
// the half of its own KV head.
//
// Data flow per tile (all in one CTA per SM):
//   loader warps 8-11 wait for a tile's raw E4M3 rows in an NS-stage ring
//                     (page size 1: gathered by the softmax warps, below; page
//                     size 64: one TMA tile load per page for K and one for
//                     V, issued here), then E4M3 -> fp16 into 128-byte-
//                     swizzled tiles (K and V, NF buffers); at a request's
//                     first tile they also write its A operand into tensor
//                     memory.
//   MMA warp 12       S(i) = A . K(i)^T into tensor memory (double-buffered),
//                     then O += P(i-1) . V(i-1) with P read from tensor memory.
//   softmax warps 0-7 two threads per row (warps w and w + 4 share the
//                     tensor-memory lanes of rows 32 (w % 4) .. + 31): warp
//                     w takes the tiles of parity w / 4, all 64 keys, and runs
//                     its own online softmax over them (own running max and
//                     sum, own O accumulator O_par, lazy rescaling: O_par is
//                     rescaled in tensor memory only when its max grows by
//                     more than 2^8), P as fp16 back into the S columns; the
//                     two work on consecutive tiles at the same time.  At a
//                     request's last tile they merge (m, l) through shared
//                     memory and each writes half the dims of a0 O_0 + a1 O_1
//                     to the partial.  With page size 1 each parity group also
//                     issues the cp.async gathers of tile i + NS - 1 once it
//                     has taken tile i (more warps issuing gathers raise the
//                     rate at which random rows arrive).
// Synchronisation by mbarriers; every wait is bounded (an expired wait sets
// the step's error word and the CTA winds down, waits for its MMAs and frees
// its tensor memory).
#pragma once

#include <cuda.h>

#include "gad_kernels.cuh"
#include "gad_tc.cuh"

namespace gad {
namespace vtc {

constexpr int TK = 64;                        // keys per tile
constexpr int SOFT = 256;                     // softmax threads: warps 0-7, two per row
constexpr int THREADS = 416;                  // 13 warps
constexpr int LOAD_T0 = SOFT;                 // first loader thread (warp 8)
constexpr int LOAD_W0 = LOAD_T0 / 32;
constexpr int LOADERS = 128;
constexpr int MMA_WARP = 12;
constexpr int RAW_STAGE = 2 * TK * ROWB;      // 16 KB: 64 K rows then 64 V rows (E4M3)
constexpr int HALF_TILE = TK * 128;           // one head of a converted tile: 64 keys x 64 fp16
constexpr int F16_TILE = 2 * HALF_TILE;       // both heads: 16 KB
constexpr int F16_BUF = 2 * F16_TILE;         // K tile then V tile: 32 KB
// Converted K/V tiles in flight.  Three, so that converting tile i waits only
// for P.V of tile i - 3: with two, the chain "P.V(i - 2) done -> convert tile
// i -> S(i) issued -> P.V(i - 1) issued (after S(i), in MMA order) -> P.V(i - 1)
// done -> convert tile i + 1" put a whole conversion and two MMA groups in
// series for every tile.
constexpr int NF = 3;
constexpr uint32_t TM_COLS = 512;             // tensor-memory columns allocated
constexpr uint32_t TM_Q = 0;                  // A operand (fp16 pairs) of even items: 64 columns
constexpr uint32_t TM_Q1 = 192;               // A operand of odd items (an item's A may be written
                                              // while the previous item's last S MMAs still read theirs)
constexpr uint32_t TM_S = 64;                 // S buffer b at TM_S + 64 b (P aliases its first 32)
constexpr uint32_t TM_O = 256;                // O_0, O_1 (even / odd tiles), 128 columns each
constexpr uint32_t TM_O_HALF = 128;           // (head 0 dims | head 1 dims)
constexpr float RESCALE_LOG2 = 8.f;           // lazy rescale threshold (P stays <= 2^8)

// mbarrier indices
constexpr int BAR_KV_READY = 0;   // [NF] converted tile (and A operand) ready  (128 loader arrivals)
constexpr int BAR_KV_FREE = 3;    // [NF] PV of the tile done: buffers free      (MMA commit)
constexpr int BAR_S_FULL = 6;     // [2] S of the tile in tensor memory          (MMA commit)
constexpr int BAR_P_FULL = 8;     // [2] P of the tile in tensor memory          (128 softmax arrivals)
constexpr int BAR_O_FREE = 10;    // O read out at a request's last tile         (256 softmax arrivals)
constexpr int BAR_MMA_DONE = 11;  // teardown: all MMAs done                     (MMA commit)
constexpr int BAR_PAIR = 12;      // [4] softmax pair qd posted both parities' (max, sum) at a request's end (64)
constexpr int BAR_RAW = 16;       // [NS] the tile's K and V rows landed (TMA bytes, or 128 gathers' arrivals)
constexpr int NBARS = 16;         // + NS

template <int NS>
struct Cfg {
    static constexpr size_t F16_BYTES = NF * F16_BUF;
    static constexpr size_t RAW_BYTES = static_cast<size_t>(NS) * RAW_STAGE;
    static constexpr int IDX_SLOTS = 2 * NS;
    static constexpr size_t IDX_BYTES = static_cast<size_t>(IDX_SLOTS) * TK * 4;
    static constexpr size_t CTRL_BYTES = 256;  // barriers, tensor-memory base, abort flag
    // softmax pairs at a request's end: [2 (request parity)][max, sum][2 (tile parity)][128 rows]
    static constexpr size_t RED_BYTES = 2 * 2 * 2 * 128 * 4;
    // + 1024 so the swizzled tiles can start on a 1024-byte boundary
    static size_t smem_bytes(int B) {
        return 1024 + F16_BYTES + RAW_BYTES + IDX_BYTES + CTRL_BYTES + RED_BYTES +
               static_cast<size_t>(4 * B + 1) * 4;
    }
    static_assert(NS >= 3, "stages");
    static_assert((NBARS + NS) * 8 + 8 <= static_cast<int>(CTRL_BYTES), "control block");
};


// Warp-uniform version: the warp continues only if every lane saw the phase.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    const bool ok = wait_bounded(bar, parity, abort_flag);
    return __all_sync(0xffffffffu, ok);
}

}  // namespace vtc

// MULTI: more than one head group (see decode_kernel).
template <int PS, int NS, bool MULTI>
// kmap, vmap (page size 64): the K and V caches as 2D tensors of 128 ngrp-byte
// rows, read one 64-row page per TMA tile load (unused for page size 1).
__global__ void __launch_bounds__(vtc::THREADS, 1)
    verify_tc_kernel(const StepParams p, const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap) {
    using namespace vtc;
    using C = Cfg<NS>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint8_t* f16 = smem;                                     // [NF][K,V][head][64 keys][128 B]
    uint8_t* raw = smem + C::F16_BYTES;                      // [NS][K rows, V rows]
    int* idx_smem = reinterpret_cast<int*>(raw + C::RAW_BYTES);
    uint8_t* ctrl = reinterpret_cast<uint8_t*>(idx_smem) + C::IDX_BYTES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + (NBARS + NS) * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl + (NBARS + NS) * 8 + 4);
    float* red = reinterpret_cast<float*>(ctrl + C::CTRL_BYTES);  // the pairs' (max, sum) at a request's end
    int* tpre = reinterpret_cast<int*>(ctrl + C::CTRL_BYTES + C::RED_BYTES);
    int* rlo = tpre + p.NB + 1;
    int* rhi = rlo + p.NB;
    int* rnew = rhi + p.NB;

    const int tid = threadIdx.x, warp = tid >> 5;
    // B counts list items (request, head group); b below is an item index.
    const int B = MULTI ? p.NB : p.B, ng = MULTI ? p.ngrp : 1;

    int total, per, t0, t1;
    build_tile_list<TK, MULTI>(p, tpre, rlo, rhi, rnew, THREADS, total, per, t0, t1);
    if (t0 >= t1) return;

    const uint32_t bar0 = smem_addr(ctrl);
    auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    if (tid == 0) {
        for (int f = 0; f < NF; ++f) {
            mbar_init(BAR(BAR_KV_READY + f), LOADERS);
            mbar_init(BAR(BAR_KV_FREE + f), 1);
        }
        mbar_init(BAR(BAR_S_FULL), 1);
        mbar_init(BAR(BAR_S_FULL + 1), 1);
        mbar_init(BAR(BAR_P_FULL), SOFT / 2);
        mbar_init(BAR(BAR_P_FULL + 1), SOFT / 2);
        mbar_init(BAR(BAR_O_FREE), SOFT);
        mbar_init(BAR(BAR_MMA_DONE), 1);
        for (int q = 0; q < 4; ++q) mbar_init(BAR(BAR_PAIR + q), 64);
        // raw stages: the TMA page loads' bytes (one arrival), or the
        // gathers of one softmax parity group (128 tracked arrivals)
        for (int st = 0; st < NS; ++st) mbar_init(BAR(BAR_RAW + st), PS == 64 ? 1 : SOFT / 2);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == MMA_WARP) {
        tc_alloc(smem_addr(tmem_slot), TM_COLS);
        tc_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // ---- tile cursors over the list (item b owns tiles [tpre[b], tpre[b+1])) ----
    auto find_req = [&](int tau) {
        int lo = 0, hi = B;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (tpre[mid] <= tau) lo = mid;
            else hi = mid;
        }
        return lo;
    };
    auto tile_k0 = [&](int tau, int b) { return (rlo[b] / TK + (tau - tpre[b])) * TK; };
    const float C2 = __ldg(p.k_scale) * 0.125f * 1.4426950408889634f;  // raw score -> log2 units

    bool prep_done = false;
    auto ensure_prep = [&]() {
        if (!prep_done) {
            pdl_wait_primary();
            prep_done = true;
        }
    };
    // A cursor over the tile list that keeps its item's data in registers:
    // shared memory is read only when it enters a new item (a chain of
    // dependent shared-memory reads per tile slowed the loaders).
    struct Cur {
        int tau, b, end, k0, lo, hi, rnew;
        const int32_t* pt;  // page-table row of the item's request
        size_t gofs;        // byte offset of the item's head group in a cache row
    };
    auto cur_enter = [&](Cur& c) {  // c.tau and c.b set
        c.end = tpre[c.b + 1];
        c.lo = rlo[c.b];
        c.hi = rhi[c.b];
        c.rnew = rnew[c.b];
        c.k0 = (c.lo / TK + (c.tau - tpre[c.b])) * TK;
        const ItemRef it = item_ref<MULTI>(p, c.b);
        c.pt = p.page_table + static_cast<size_t>(it.req) * p.max_pages;
        c.gofs = static_cast<size_t>(it.grp) * ROWB;
    };
    auto cur_init = [&](Cur& c, int tau) {
        c.tau = tau;
        c.b = find_req(tau);
        cur_enter(c);
    };
    auto cur_next = [&](Cur& c) {
        ++c.tau;
        c.k0 += TK;
        if (c.tau >= c.end && c.tau < t1 && c.b < B - 1) {
            do {
                ++c.b;
            } while (c.b < B - 1 && c.tau >= tpre[c.b + 1]);
            cur_enter(c);
        }
    };
    // rows this step writes (the prep kernel, which may still run) are read
    // only after it has finished
    auto k_needs_prep = [&](const Cur& c) { return c.k0 + TK - 1 >= c.rnew; };
    // Page size 1: the softmax warps gather the K and V rows (warps that issue
    // cp.async limit the gather rate, and the loaders have the conversion to
    // do).  One parity group (128 threads) fills one tile's raw stage: thread t
    // copies 16-byte chunk t % 8 of rows t / 8 + 16 q (q < 4) for K and V, so
    // that eight lanes cover a whole 128-byte row, then lets the stage's
    // mbarrier track its copies.
    const size_t row_pitch = static_cast<size_t>(ROWB) * ng;
    auto row_entries = [&](const Cur& c, int gt, int (&e)[4]) {  // page-table entries of the rows, or -1
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int k = c.k0 + (gt >> 3) + 16 * q;
            e[q] = (c.tau < t1 && k >= c.lo && k <= c.hi && k < p.max_pages) ? __ldg(c.pt + k) : -1;
        }
    };
    auto gather_rows = [&](const Cur& c, int gt, const int (&e)[4]) {
        if (k_needs_prep(c)) ensure_prep();
        const int jc = gt & 7;
        const uint32_t base = smem_addr(raw + ((c.tau - t0) % NS) * RAW_STAGE);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int r = (gt >> 3) + 16 * q;
            const bool ok = e[q] >= 0 && e[q] < p.num_rows;
            const size_t off = ok ? static_cast<size_t>(e[q]) * row_pitch + c.gofs + 16 * jc : 0;
            const uint32_t d = base + r * ROWB + ((jc ^ (r & 7)) << 4);
            cp_async16(d, p.k_cache + off, ok ? 16 : 0);
            cp_async16(d + TK * ROWB, p.v_cache + off, ok ? 16 : 0);
        }
        cp_async_mbar_arrive_noinc(BAR(BAR_RAW + (c.tau - t0) % NS));
    };

    if (warp >= LOAD_W0 && warp < MMA_WARP) {
        // =================== loaders: gather, convert, A operand ===================
        const int ltid = tid - LOAD_T0;
        // Page size 64: the loaders fetch each tile's page index (NS - 1 tiles
        // ahead of its load) and issue its two TMA page loads.
        auto issue_idx = [&](const Cur& c) {
            if (c.tau >= t1) return;
            int* dst = idx_smem + ((c.tau - t0) % C::IDX_SLOTS) * TK;
            if (ltid < TK / PS) {
                const int pg = c.k0 / PS + ltid;
                if (pg < p.max_pages) cp_async4(smem_addr(dst + ltid), c.pt + pg);
                else dst[ltid] = -1;
            }
        };
        int n_kv_issued = 0;  // tiles whose page loads were issued (the same count in every loader)
        auto issue_kv = [&](const Cur& c) {
            if (c.tau >= t1) return;
            if (k_needs_prep(c)) ensure_prep();
            const int* ix = idx_smem + ((c.tau - t0) % C::IDX_SLOTS) * TK;
            const uint32_t base = smem_addr(raw + ((c.tau - t0) % NS) * RAW_STAGE);
            ++n_kv_issued;
            // the tile is one page: its K and V rows by two TMA tile loads
            // (128-byte swizzle, the layout the page-size-1 gathers write); a page
            // index past the table (-1) or rows past the cache fall outside the
            // tensor and read as zeros
            if (ltid == 0) {
                const int pg = ix[0];
                const int y = pg >= 0 ? pg * PS : -PS;
                const uint32_t bar = BAR(BAR_RAW + (c.tau - t0) % NS);
                mbar_arrive_expect_tx(bar, RAW_STAGE);
                tma_load_2d(base, &kmap, static_cast<int>(c.gofs), y, bar);
                tma_load_2d(base + TK * ROWB, &vmap, static_cast<int>(c.gofs), y, bar);
            }
        };
        // A operand of item b's S MMA: row ltid = [q | 0] (KV head 0) or [0 | q].
        auto write_q = [&](int b, uint32_t qcol) {
            ensure_prep();
            const int g = ltid >> 6, j = (ltid >> 3) & 7, hh = ltid & 7;
            const ItemRef it = item_ref<MULTI>(p, b);
            uint32_t q[32], z[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) z[c] = 0u;
            if (j < it.len) {
                const uint4* src = reinterpret_cast<const uint4*>(
                    p.q_ws + (((static_cast<size_t>(it.t0) + j) * ng + it.grp) * HQ + g * GRP + hh) * HD);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v = src[c];
                    q[4 * c] = v.x;
                    q[4 * c + 1] = v.y;
                    q[4 * c + 2] = v.z;
                    q[4 * c + 3] = v.w;
                }
            } else {
#pragma unroll
                for (int c = 0; c < 32; ++c) q[c] = 0u;
            }
            const uint32_t ta = tmem + qcol + (static_cast<uint32_t>(32 * (warp - LOAD_W0)) << 16);
            tc_st32(ta + (g == 0 ? 0u : 32u), q);
            tc_st32(ta + (g == 0 ? 32u : 0u), z);
        };
        // raw stage -> fp16 tile: thread = (K or V, row r); 16 codes -> two 16-byte fp16 chunks.
        // With page size 64 whole pages arrive, so keys outside the item's range
        // [lo, hi] (slots of the page not yet written, or before a window) are
        // converted as zeros, as the page-size-1 gathers zero-fill them.
        auto convert = [&](int stage, int buf, int k0, int lo, int hi) {
            const int kv = ltid >> 6, r = ltid & 63;
            const uint32_t src = smem_addr(raw + stage * RAW_STAGE) + kv * TK * ROWB + r * ROWB;
            const uint32_t dst = smem_addr(f16 + buf * F16_BUF) + kv * F16_TILE + r * 128;
            uint4 w[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) w[j] = lds128(src + ((j ^ (r & 7)) << 4));
            if (PS == 64 && (k0 + r < lo || k0 + r > hi)) {
#pragma unroll
                for (int j = 0; j < 8; ++j) w[j] = make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t row = dst + (j >> 2) * HALF_TILE;
                const int c0 = 2 * (j & 3);
                uint4 a, b;
                a.x = e4m3x2_to_f16x2(w[j].x);
                a.y = e4m3x2_to_f16x2(w[j].x >> 16);
                a.z = e4m3x2_to_f16x2(w[j].y);
                a.w = e4m3x2_to_f16x2(w[j].y >> 16);
                b.x = e4m3x2_to_f16x2(w[j].z);
                b.y = e4m3x2_to_f16x2(w[j].z >> 16);
                b.z = e4m3x2_to_f16x2(w[j].w);
                b.w = e4m3x2_to_f16x2(w[j].w >> 16);
                sts128(row + ((c0 ^ (r & 7)) << 4), a);
                sts128(row + (((c0 + 1) ^ (r & 7)) << 4), b);
            }
        };

        Cur xc, kc, cc;  // page-index cursor (NS - 1 tiles ahead), page-load cursor, current tile
        cur_init(xc, t0);
        kc = xc;
        cc = xc;
        if (PS == 64) {
            for (int d = 0; d < NS - 1; ++d) {
                issue_idx(xc);
                cur_next(xc);
            }
            cp_async_commit();
            cp_async_wait<0>();
            bar_red_or(1, LOADERS, false);
            for (int d = 0; d < NS - 1; ++d) {
                issue_kv(kc);
                cur_next(kc);
                issue_idx(xc);
                cur_next(xc);
                cp_async_commit();
            }
        }
        int seg_b = -1, nseg = 0, seg_i0 = 0;  // current item, items begun, its first tile
        const int n_tiles = t1 - t0;
        int i = 0;
        for (; i < n_tiles; ++i) {
            if (PS == 64) cp_async_wait<NS - 2>();  // the page indices NS - 1 tiles ahead
            const int cb = cc.b;
            const bool seg_start = cb != seg_b;
            // A new item's A operand is written before the waits below (its q
            // load then overlaps them) when its buffer is known to be free: the
            // first two items' buffers are fresh; else the buffer's last reader,
            // the S MMA of the previous item's predecessor's last tile (<= i - 3
            // when the previous item had two tiles or more), is done once PV(i - 4)
            // is, which the wait of tile i - 1 saw.
            const bool early_q = seg_start && (nseg < 2 || (seg_i0 <= i - 2 && i >= NF + 1));
            if (early_q) write_q(cb, (nseg & 1) ? TM_Q1 : TM_Q);
            // tile i's raw stage filled (page loads, or the softmax warps' gathers)
            bool bad = !wait_bounded(BAR(BAR_RAW + i % NS), (i / NS) & 1, abort_flag);
            // buffers i % NF are free once PV(i - NF) is done, which also means every
            // S MMA up to tile i - NF + 1 is done: the A operand this item takes
            // (the one of the item before the previous) is no longer read.  Tile 2
            // has no such wait; if it starts a third item, S(0) (item 0's) must be done.
            if (i >= NF && !bad) bad = !wait_bounded(BAR(BAR_KV_FREE + i % NF), ((i - NF) / NF) & 1, abort_flag);
            static_assert(NF == 3, "the A-operand wait below assumes three buffers");
            if (i == 2 && seg_start && nseg >= 2 && !bad) bad = !wait_bounded(BAR(BAR_S_FULL), 0, abort_flag);
            // past this barrier: every loader has converted tile i - 1, so its raw
            // stage may be refilled
            if (bar_red_or(1, LOADERS, bad)) break;
            if (seg_start) {
                if (!early_q) write_q(cb, (nseg & 1) ? TM_Q1 : TM_Q);
                seg_b = cb;
                seg_i0 = i;
                ++nseg;
            }
            convert(i % NS, i % NF, cc.k0, cc.lo, cc.hi);
            fence_proxy_async_smem();
            if (seg_start) {
                tc_wait_st();
                tc_fence_before();
            }
            mbar_arrive(BAR(BAR_KV_READY + i % NF));
            // page loads for tile i + NS - 1 (into the stage of tile i - 1), off the
            // path from "buffer free" to "tile ready"
            if (PS == 64) {
                issue_kv(kc);
                cur_next(kc);
                issue_idx(xc);
                cur_next(xc);
                cp_async_commit();
            }
            cur_next(cc);
        }
        cp_async_wait<0>();
        if (PS == 64 && ltid == 0) {
            // every page load issued lands before the CTA leaves (its shared
            // memory is the destination); without an abort they all have
            for (int tile = i; tile < n_kv_issued; ++tile)
                wait_bounded(BAR(BAR_RAW + tile % NS), (tile / NS) & 1, abort_flag, false, TEARDOWN_LIMIT_NS);
        }
    }
    else if (warp == MMA_WARP) {
        // =================== MMA issue (whole warp, one elected lane issues) ===================
        // The warp runs the control flow together so that every operand of the
        // MMA and commit instructions is warp-uniform.
        constexpr uint32_t ID_S = idesc_f16_f32(128, TK, 0);  // S: A . K^T, K-major B
        constexpr uint32_t ID_O = idesc_f16_f32(128, 128, 1);  // O: P . V, MN-major B, both heads' dims
        const uint32_t f16_base = smem_addr(f16);
        // O_(k & 1) += P(k) . V(k) over both KV heads' dims at once (N = 128:
        // the two heads' V tiles are the MN-major operand's two 64-wide atoms,
        // HALF_TILE bytes apart; each row keeps its own head's half); `pos` is
        // k's index within its request (the first tile of each parity overwrites).
        auto issue_pv = [&](int k, int pos, int seg) {
            if (!wait_warp(BAR(BAR_P_FULL + (k & 1)), (k >> 1) & 1, abort_flag)) return false;
            if (pos == 0 && seg >= 1 && !wait_warp(BAR(BAR_O_FREE), (seg - 1) & 1, abort_flag)) return false;
            tc_fence_after();
            const uint32_t vb = f16_base + (k % NF) * F16_BUF + F16_TILE;
            const uint32_t pa = tmem + TM_S + 64u * (k & 1);
            const uint32_t av[4] = {pa, pa + 8u, pa + 16u, pa + 24u};
            const uint64_t bd[4] = {smem_desc_sw128_mn2(vb, HALF_TILE), smem_desc_sw128_mn2(vb + 2048, HALF_TILE),
                                    smem_desc_sw128_mn2(vb + 4096, HALF_TILE), smem_desc_sw128_mn2(vb + 6144, HALF_TILE)};
            tc_mma_ts4(tmem + TM_O + TM_O_HALF * (k & 1), av, bd, ID_O, pos >= 2 ? 1u : 0u);
            tc_commit(BAR(BAR_KV_FREE + k % NF));
            return true;
        };
        int ct = t0, cb = find_req(t0);
        int cb_end = tpre[cb + 1];             // first tile past item cb (kept in a register)
        int seg_b = -1, seg = -1, seg_i0 = 0;  // current request, its count and first tile here
        int prev_pos = 0;
        int prev_seg = -1;
        bool ok = true;
        int i = 0;
        for (; ct < t1; ++i) {
            if (cb != seg_b) {
                seg_b = cb;
                ++seg;
                seg_i0 = i;
            }
            if (!wait_warp(BAR(BAR_KV_READY + i % NF), (i / NF) & 1, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t kbuf = f16_base + (i % NF) * F16_BUF;
            const uint32_t sd = tmem + TM_S + 64u * (i & 1);
#pragma unroll
            for (int hk = 0; hk < 2; ++hk) {  // the contraction's two KV-head halves, 4 K16 steps each
                const uint32_t qa = tmem + ((seg & 1) ? TM_Q1 : TM_Q) + 32u * hk;
                const uint32_t aq[4] = {qa, qa + 8u, qa + 16u, qa + 24u};
                const uint32_t kb = kbuf + hk * HALF_TILE;
                const uint64_t bd[4] = {smem_desc_sw128(kb), smem_desc_sw128(kb + 32),
                                        smem_desc_sw128(kb + 64), smem_desc_sw128(kb + 96)};
                tc_mma_ts4(sd, aq, bd, ID_S, hk > 0 ? 1u : 0u);
            }
            tc_commit(BAR(BAR_S_FULL + (i & 1)));
            if (i > 0 && !issue_pv(i - 1, prev_pos, prev_seg)) {
                ok = false;
                break;
            }
            prev_pos = i - seg_i0;
            prev_seg = seg;
            if (++ct >= cb_end && ct < t1) {
                while (cb < B - 1 && ct >= tpre[cb + 1]) ++cb;
                cb_end = tpre[cb + 1];
            }
        }
        if (ok && i > 0) issue_pv(i - 1, prev_pos, prev_seg);
        // every MMA this warp issued is done before the tensor memory is freed
        tc_commit(BAR(BAR_MMA_DONE));
        const bool done = wait_bounded(BAR(BAR_MMA_DONE), 0, abort_flag, false, TEARDOWN_LIMIT_NS);
        __syncwarp();
        (void)done;
    } else {
        // =================== softmax: two threads per row ===================
        // Warps w and w + 4 share the tensor-memory lanes of rows 32 (w % 4) ..
        // + 31; warp w takes the tiles of parity par = w / 4 (all 64 keys) with
        // its own running max, sum and O accumulator, so the two work on
        // consecutive tiles at once and never wait for each other until a
        // request's last tile, where they merge through shared memory
        // (double-buffered by request parity) after meeting at the pair's
        // mbarrier (a bounded wait, as every other).
        const int par = warp >> 2, qd = warp & 3;
        const int r = 32 * qd + (tid & 31);
        const int g = r >> 6, j = (r >> 3) & 7, qh = g * GRP + (r & 7);
        const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
        const uint32_t o_own = tmem + TM_O + TM_O_HALF * par + 64u * g + lane_base;  // O_par, this row's head
        int ct = t0, cb = find_req(t0);
        int seg_b = -1, seg_t1 = 0, k0 = 0;  // current request, end of its tiles here, tile key
        float m_run = -INFINITY, l_run = 0.f;  // running max (raw score units) and sum over this parity's tiles
        int lo_j = INT_MAX, hi_j = -1;
        int seg_len = 0;  // tokens of the current item
        int n_end = 0;    // requests finished here
        // page size 1: this group gathers tiles par, par + 2, .. below NS - 1
        // now, and tile i + NS - 1 once it has taken tile i (whose S MMA being
        // done means tile i - 1 is converted, so that stage is free)
        const int gt = tid & 127;
        Cur gc;
        int pend[4] = {-1, -1, -1, -1};  // page-table entries of this thread's rows in tile gc, loaded a tile early
        if (PS == 1) {
            for (int T = par; T < NS - 1 && t0 + T < t1; T += 2) {
                cur_init(gc, t0 + T);
                row_entries(gc, gt, pend);
                gather_rows(gc, gt, pend);
            }
            if (t0 + par + NS - 1 < t1) {
                cur_init(gc, t0 + par + NS - 1);
                row_entries(gc, gt, pend);
            } else {
                gc.tau = t1;
            }
        }
        // the position of this row's token in an item, requested one item ahead
        // (a global load at each item's first tile would sit on the path)
        auto load_pos = [&](int b) {
            const ItemRef it = item_ref<MULTI>(p, b);
            return j < it.len ? p.positions[static_cast<size_t>(it.t0) + j] : int64_t{-1};
        };
        int pf_b = cb;
        int64_t pf_pos = load_pos(cb);
        for (int i = 0; ct < t1; ++i) {
            const bool seg_start = cb != seg_b;
            if (seg_start) {
                seg_b = cb;
                seg_t1 = min(t1, tpre[cb + 1]);
                k0 = tile_k0(ct, cb);
                m_run = -INFINITY;
                l_run = 0.f;
                const ItemRef it = item_ref<MULTI>(p, cb);
                seg_len = it.len;
                const int64_t pos64 = pf_b == cb ? pf_pos : load_pos(cb);
                if (seg_t1 < t1) {
                    pf_b = cb + 1;
                    pf_pos = load_pos(cb + 1);
                }
                if (j < it.len) {
                    const int pos = static_cast<int>(pos64);
                    hi_j = pos;
                    lo_j = p.window > 0 ? max(0, pos - p.window + 1) : 0;
                } else {
                    lo_j = INT_MAX;
                    hi_j = -1;
                }
            } else {
                k0 += TK;
            }
            const bool seg_end = ct + 1 >= seg_t1;

            if ((i & 1) == par) {
                if (!wait_warp(BAR(BAR_S_FULL + par), (i >> 1) & 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t sbuf = tmem + TM_S + 64u * par + lane_base;
                const int cmin = lo_j == INT_MAX ? TK : lo_j - k0;
                const int cmax = hi_j - k0;
                const bool full = cmin <= 0 && cmax >= TK - 1;
                uint32_t sr[32];
                // pass 1: the row's max over the tile's 64 keys (two 32-column loads)
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    tc_ld32(sbuf + 32u * ch, sr);
                    tc_wait_ld();
                    if (!full) {
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            if (32 * ch + c < cmin || 32 * ch + c > cmax) sr[c] = __float_as_uint(-INFINITY);
                    }
#pragma unroll
                    for (int c = 0; c < 32; c += 8) {
                        m4[c >> 3] = fmax3(m4[c >> 3], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
                        m4[c >> 3] = fmax3(m4[c >> 3], __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
                        m4[c >> 3] = fmax3(m4[c >> 3], __uint_as_float(sr[c + 4]), __uint_as_float(sr[c + 5]));
                        m4[c >> 3] = fmax3(m4[c >> 3], __uint_as_float(sr[c + 6]), __uint_as_float(sr[c + 7]));
                    }
                }
                const float mx = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]);
                // lazy rescale: O_par (in tensor memory) is corrected only when
                // this warp's max grows a lot
                const float m_new = fmaxf(m_run, mx);
                bool corr = false;
                if (m_new > m_run) {
                    if (m_run == -INFINITY || (m_new - m_run) * C2 <= RESCALE_LOG2) {
                        if (m_run == -INFINITY) m_run = m_new;
                    } else {
                        corr = true;
                    }
                }
                bool bad = false;
                if (__any_sync(0xffffffffu, corr)) {
                    // P.V of this warp's previous tile (i - 2, same request) must be
                    // done before O_par is touched
                    const bool ok = wait_warp(BAR(BAR_KV_FREE + (i - 2) % NF), ((i - 2) / NF) & 1, abort_flag);
                    const float alpha = corr ? fast_exp2((m_run - m_new) * C2) : 1.f;
                    if (ok) {
                        tc_fence_after();
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            uint32_t o[32];
                            tc_ld32(o_own + 32u * q, o);
                            tc_wait_ld();
#pragma unroll
                            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                            tc_st32(o_own + 32u * q, o);
                        }
                        tc_wait_st();
                    }
                    bad = !ok;
                    if (corr) {
                        l_run *= alpha;
                        m_run = m_new;
                    }
                }
                if (bad) break;
                // pass 2: P = 2^(s - m) for each 32-key chunk, written as fp16 over the
                // S columns already read (keys 32 ch .. -> columns 16 ch ..)
                const float mc = m_run == -INFINITY ? 0.f : m_run * C2;
                float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    tc_ld32(sbuf + 32u * ch, sr);
                    tc_wait_ld();
                    if (!full) {
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            if (32 * ch + c < cmin || 32 * ch + c > cmax) sr[c] = __float_as_uint(-INFINITY);
                    }
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const float p0 = fast_exp2(fmaf(__uint_as_float(sr[2 * c]), C2, -mc));
                        const float p1 = fast_exp2(fmaf(__uint_as_float(sr[2 * c + 1]), C2, -mc));
                        l4[c & 3] += p0 + p1;
                        pk[c] = pack_f16x2(p0, p1);
                    }
                    tc_st16(sbuf + 16u * ch, pk);
                }
                l_run += (l4[0] + l4[1]) + (l4[2] + l4[3]);
                tc_wait_st();
                tc_fence_before();
                mbar_arrive(BAR(BAR_P_FULL + par));
                if (PS == 1 && gc.tau < t1) {
                    gather_rows(gc, gt, pend);
                    cur_next(gc);
                    cur_next(gc);
                    row_entries(gc, gt, pend);
                }
            }

            if (seg_end) {
                // the request's last P.V (in MMA order, every earlier one too) done
                const bool ok = wait_warp(BAR(BAR_KV_FREE + i % NF), (i / NF) & 1, abort_flag);
                float* rm = red + (n_end & 1) * 512;  // [max, sum][parity][row]
                rm[par * 128 + r] = m_run == -INFINITY ? -INFINITY : m_run * C2;
                rm[256 + par * 128 + r] = l_run;
                mbar_arrive(BAR(BAR_PAIR + qd));  // both warps' (max, sum) posted
                if (!ok || !wait_warp(BAR(BAR_PAIR + qd), n_end & 1, abort_flag)) break;
                ++n_end;
                const float m0 = rm[r], m1 = rm[128 + r];
                const float m = fmaxf(m0, m1);
                // a parity with no tile of this request (or only masked keys) has
                // weight 0; its accumulator may hold another request's values
                const float a0 = m0 == -INFINITY ? 0.f : fast_exp2(m0 - m);
                const float a1 = m1 == -INFINITY ? 0.f : fast_exp2(m1 - m);
                const float l = a0 * rm[256 + r] + a1 * rm[384 + r];
                tc_fence_after();
                // dims 32 par .. + 31 of this row's head from both accumulators
                const uint32_t oa = tmem + TM_O + 64u * g + 32u * par + lane_base;
                uint32_t o0[32], o1[32];
                tc_ld32(oa, o0);
                tc_ld32(oa + TM_O_HALF, o1);
                tc_wait_ld();
                if (j < seg_len) {
                    const size_t slot = static_cast<size_t>(blockIdx.x) + cb;
                    const size_t base = (slot * p.lt + j) * HQ + qh;
                    float4* dst = reinterpret_cast<float4*>(p.part_o + base * HD + 32 * par);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        float v[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float x0 = a0 != 0.f ? a0 * __uint_as_float(o0[4 * q + e]) : 0.f;
                            const float x1 = a1 != 0.f ? a1 * __uint_as_float(o1[4 * q + e]) : 0.f;
                            v[e] = x0 + x1;
                        }
                        dst[q] = make_float4(v[0], v[1], v[2], v[3]);
                    }
                    if (par == 0) {
                        p.part_ml[base * 2 + 0] = m;
                        p.part_ml[base * 2 + 1] = l;
                    }
                }
                tc_fence_before();
                mbar_arrive(BAR(BAR_O_FREE));
            }
            ++ct;
            if (seg_end)
                while (cb < B - 1 && ct >= tpre[cb + 1]) ++cb;
        }
        cp_async_wait<0>();  // every gather this thread issued has landed before the CTA leaves
    }

    // ---- teardown ----
    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tc_dealloc(tmem, TM_COLS);
    }
    if (tid == 0 && *abort_flag) {
        pdl_wait_primary();  // the step's first kernel has cleared the status word
        atomicOr(p.status, STATUS_ATTN_WAIT);
    }
    pdl_launch_dependents();
}

}  // namespace gad
